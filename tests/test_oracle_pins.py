"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

The pages print no worked numeric example for this operator, so the oracle is
pinned by closed forms, textbook special cases, brute force on tiny inputs and
invariants that the mathematics fixes.  Each pin is chosen so that a plausible
mistake (a swapped band, a wrong rotation sign, RoPE in the denominator, eps
inside the dot product, a transposed state, a block that cannot see itself)
makes at least one of them fail.
"""
import math

import numpy as np
import pytest

import oracle as orc
from gated_linear_attention_relu_b200 import workloads as wl


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# --------------------------------------------------------------------------
# RoPE: closed forms and the properties of a rotation
# --------------------------------------------------------------------------

def test_band_frequencies_decimal_closed_form():
    # base 10000, band width 8: base**(-2i/8) = 10**(-i).
    th = orc.band_frequencies(8, 10000.0)
    assert np.allclose(th, [1.0, 0.1, 0.01, 0.001], rtol=1e-15, atol=0)


def test_grid_positions_row_major_time_slowest():
    pos = orc.grid_positions(2, 3, 5)
    assert pos.shape == (30, 3)
    for n, expect in [(0, (0, 0, 0)), (4, (0, 0, 4)), (5, (0, 1, 0)), (14, (0, 2, 4)),
                      (15, (1, 0, 0)), (29, (1, 2, 4))]:
        assert tuple(pos[n]) == expect


@pytest.mark.parametrize("channel,angle,pair", [
    (0, 3.0, (0, 1)),      # t band, pair 0, theta 1, t = 3
    (2, 0.3, (2, 3)),      # t band, pair 1, theta 0.1, t = 3
    (10, 0.5, (10, 11)),   # h band (offset 8), pair 1, theta 0.1, h = 5
    (22, 0.007, (22, 23)), # w band (offset 16), pair 3, theta 0.001, w = 7
])
def test_rope_unit_vectors_closed_form(channel, angle, pair):
    # bands (8, 8, 8), base 10000 -> theta = 1, 0.1, 0.01, 0.001 in every band.
    pos = np.array([[3, 5, 7]])
    x = np.zeros((1, 24))
    x[0, channel] = 1.0
    y = orc.rope3d(x, pos, (8, 8, 8), 10000.0)[0]
    expect = np.zeros(24)
    # The first channel of a pair goes to (cos a, sin a): counter-clockwise rotation.
    expect[pair[0]] = math.cos(angle)
    expect[pair[1]] = math.sin(angle)
    assert np.allclose(y, expect, atol=1e-15)
    # The second channel of the pair goes to (-sin a, cos a).
    x2 = np.zeros((1, 24))
    x2[0, pair[1]] = 1.0
    y2 = orc.rope3d(x2, pos, (8, 8, 8), 10000.0)[0]
    expect2 = np.zeros(24)
    expect2[pair[0]] = -math.sin(angle)
    expect2[pair[1]] = math.cos(angle)
    assert np.allclose(y2, expect2, atol=1e-15)


def test_rope_matches_complex_multiplication():
    # RoFormer's complex form: pair (x0, x1) as x0 + i x1, multiplied by exp(i * pos * theta).
    rng = np.random.default_rng(1)
    bands = (4, 6, 6)
    x = _rand(rng, 20, 16)
    pos = rng.integers(0, 50, size=(20, 3))
    y = orc.rope3d(x, pos, bands, 100.0)
    off = 0
    for axis, D in enumerate(bands):
        for i in range(D // 2):
            theta = 100.0 ** (-2.0 * i / D)
            zc = (x[:, off + 2 * i] + 1j * x[:, off + 2 * i + 1]) * np.exp(1j * pos[:, axis] * theta)
            assert np.allclose(y[:, off + 2 * i], zc.real, atol=1e-12)
            assert np.allclose(y[:, off + 2 * i + 1], zc.imag, atol=1e-12)
        off += D


def test_rope_norm_identity_relative_composition():
    rng = np.random.default_rng(2)
    bands = (8, 12, 12)
    x = _rand(rng, 64, 32)
    y = _rand(rng, 64, 32)
    p = rng.integers(0, 300, size=(64, 3))
    p2 = rng.integers(0, 300, size=(64, 3))
    rx = orc.rope3d(x, p, bands, 10000.0)
    # norm preservation
    assert np.allclose(np.linalg.norm(rx, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    # identity at position 0
    assert np.array_equal(orc.rope3d(x, np.zeros_like(p), bands, 10000.0), x)
    # relative property: R(p)x . R(p')y = x . R(p'-p)y
    lhs = np.sum(rx * orc.rope3d(y, p2, bands, 10000.0), axis=1)
    rhs = np.sum(x * orc.rope3d(y, p2 - p, bands, 10000.0), axis=1)
    assert np.allclose(lhs, rhs, rtol=1e-10, atol=1e-10)
    # composition: R(p') R(p) = R(p + p')
    assert np.allclose(orc.rope3d(rx, p2, bands, 10000.0), orc.rope3d(x, p + p2, bands, 10000.0),
                       atol=1e-11)


# --------------------------------------------------------------------------
# The operator: brute force, closed forms, special cases, invariants
# --------------------------------------------------------------------------

def test_linear_form_equals_brute_form_on_tiny_workload():
    w = wl.WORKLOADS["tiny_f32"]
    Q, K, V, G = (t.double().numpy() for t in wl.generate(w, "cpu"))
    O = orc.forward_bidir(Q, K, V, G, (w.T, w.Hh, w.W), w.bands, w.rope_base, w.eps)
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    for h in range(w.H):
        ob = orc.forward_brute(Q[0, h], K[0, h], V[0, h], G[0, h], pos, w.bands, w.rope_base, w.eps)
        assert np.max(np.abs(ob - O[0, h])) <= 1e-12 * np.max(np.abs(ob))


@pytest.mark.parametrize("grid,d,bands", [((3, 5, 7), 16, (4, 6, 6)), ((4, 4, 32), 32, (8, 12, 12)),
                                          ((1, 1, 1), 8, (2, 2, 4)), ((7, 1, 3), 32, (0, 16, 16))])
def test_linear_form_equals_brute_form_random_grids(grid, d, bands):
    rng = np.random.default_rng(sum(grid) + d)
    N = grid[0] * grid[1] * grid[2]
    q, k, v, g = (_rand(rng, 1, 1, N, d) for _ in range(4))
    O = orc.forward_bidir(q, k, v, g, grid, bands, 500.0, 1e-6)[0, 0]
    ob = orc.forward_brute(q[0, 0], k[0, 0], v[0, 0], g[0, 0], orc.grid_positions(*grid), bands,
                           500.0, 1e-6)
    assert np.max(np.abs(ob - O)) <= 1e-11 * np.max(np.abs(ob))


def test_single_token_closed_form_and_eps_placement():
    # N = 1: the rotation cancels (same position), so o = (q+.k+)/(q+.k+ + eps) v sigmoid(g).
    d = 8
    q = np.zeros((1, 1, 1, d)); k = np.zeros((1, 1, 1, d))
    q[..., 3] = 1e-3; q[..., 5] = -2.0  # the negative entry is cut by ReLU
    k[..., 3] = 1e-3; k[..., 5] = 7.0
    v = np.arange(1.0, d + 1).reshape(1, 1, 1, d)
    g = np.full((1, 1, 1, d), 0.3)
    eps = 1e-6
    O = orc.forward_bidir(q, k, v, g, (1, 1, 1), (2, 2, 4), 10000.0, eps)[0, 0, 0]
    dot = 1e-6  # q+ . k+ = 1e-3 * 1e-3
    expect = dot / (dot + eps) * np.arange(1.0, d + 1) / (1.0 + math.exp(-0.3))
    assert np.allclose(O, expect, rtol=1e-14)
    assert np.allclose(O, 0.5 * np.arange(1.0, d + 1) / (1.0 + math.exp(-0.3)), rtol=1e-14)


def test_two_token_numerator_rotated_denominator_not():
    # q = k_m = e0 (t band pair 0, theta 1) at t = 0 and t = 1.
    d = 8
    bands = (2, 2, 4)
    q = np.zeros((1, 1, 2, d)); k = np.zeros((1, 1, 2, d))
    q[..., 0] = 1.0; k[..., 0] = 1.0
    a = np.array([1.0, -2.0, 3.0, 0.5, 0.0, 4.0, -1.0, 2.0])
    b = np.array([0.0, 1.0, -1.0, 2.0, 5.0, -3.0, 1.0, 1.0])
    v = np.stack([a, b]).reshape(1, 1, 2, d)
    g = np.full((1, 1, 2, d), 50.0)  # sigmoid = 1 - 2e-22
    eps = 1e-6
    O = orc.forward_bidir(q, k, v, g, (2, 1, 1), bands, 10000.0, eps)[0, 0]
    c1 = math.cos(1.0)
    assert np.allclose(O[0], (a + c1 * b) / (2.0 + eps), rtol=1e-13)
    assert np.allclose(O[1], (c1 * a + b) / (2.0 + eps), rtol=1e-13)


def test_zero_angles_reduce_to_relu_linear_attention_convex_combination():
    # All positions 0: no rotation; o / sigmoid(g) is a convex combination of the
    # value rows up to eps (Katharopoulos-style ReLU linear attention).
    rng = np.random.default_rng(5)
    N, d = 50, 16
    q, k, v, g = (_rand(rng, N, d) for _ in range(4))
    pos0 = np.zeros((N, 3), dtype=np.int64)
    O = orc.forward_positions(q, k, v, g, pos0, (4, 6, 6), 10000.0, 0.0)
    r = O / orc.sigmoid(g)
    assert np.all(r <= v.max(axis=0) + 1e-12)
    assert np.all(r >= v.min(axis=0) - 1e-12)
    # and with V = 1 everywhere, o = sigmoid(g) exactly (eps = 0)
    O1 = orc.forward_positions(q, k, np.ones_like(v), g, pos0, (4, 6, 6), 10000.0, 0.0)
    assert np.allclose(O1, orc.sigmoid(g), rtol=1e-13)


def test_joint_permutation_equivariance_and_state_invariance():
    rng = np.random.default_rng(6)
    N, d, bands = 60, 16, (4, 6, 6)
    q, k, v, g = (_rand(rng, N, d) for _ in range(4))
    pos = rng.integers(0, 20, size=(N, 3))
    perm = rng.permutation(N)
    O = orc.forward_positions(q, k, v, g, pos, bands, 10000.0, 1e-6)
    Op = orc.forward_positions(q[perm], k[perm], v[perm], g[perm], pos[perm], bands, 10000.0, 1e-6)
    assert np.allclose(Op, O[perm], rtol=1e-12, atol=1e-14)
    S, z = orc.head_state(k, v, pos, bands, 10000.0)
    Sp, zp = orc.head_state(k[perm], v[perm], pos[perm], bands, 10000.0)
    assert np.allclose(S, Sp, atol=1e-12) and np.allclose(z, zp, atol=1e-12)


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_translation_invariance(axis):
    rng = np.random.default_rng(7 + axis)
    w = wl.custom("t", 1, 1, 3, 4, 5, d=16, bands=(4, 6, 6), dtype="f32")
    N = w.N
    q, k, v, g = (_rand(rng, N, 16) for _ in range(4))
    pos = orc.grid_positions(3, 4, 5)
    O = orc.forward_positions(q, k, v, g, pos, w.bands, 10000.0, 1e-6)
    shift = np.zeros(3, dtype=np.int64)
    shift[axis] = 37
    O2 = orc.forward_positions(q, k, v, g, pos + shift, w.bands, 10000.0, 1e-6)
    assert np.allclose(O, O2, rtol=1e-11, atol=1e-13)


def test_scale_invariance_in_q_and_k_and_linearity_in_v():
    rng = np.random.default_rng(8)
    N, d, bands = 40, 16, (4, 6, 6)
    q, k, v, v2, g = (_rand(rng, N, d) for _ in range(5))
    pos = rng.integers(0, 9, size=(N, 3))
    f = lambda q_, k_, v_: orc.forward_positions(q_, k_, v_, g, pos, bands, 10000.0, 0.0)
    O = f(q, k, v)
    assert np.allclose(f(3.5 * q, k, v), O, rtol=1e-12)
    assert np.allclose(f(q, 0.25 * k, v), O, rtol=1e-12)
    assert np.allclose(f(q, k, 2.0 * v - 3.0 * v2), 2.0 * O - 3.0 * f(q, k, v2), rtol=1e-10, atol=1e-12)


def test_gate_limits():
    rng = np.random.default_rng(9)
    N, d, bands = 30, 16, (4, 6, 6)
    q, k, v = (_rand(rng, N, d) for _ in range(3))
    pos = rng.integers(0, 9, size=(N, 3))
    ungated = orc.forward_positions(q, k, v, np.full((N, d), 60.0), pos, bands, 10000.0, 1e-6)
    half = orc.forward_positions(q, k, v, np.zeros((N, d)), pos, bands, 10000.0, 1e-6)
    off = orc.forward_positions(q, k, v, np.full((N, d), -800.0), pos, bands, 10000.0, 1e-6)
    assert np.allclose(half, 0.5 * ungated, rtol=1e-14)
    assert np.all(off == 0.0)


def test_denominator_positive_with_sparse_keys():
    # K shifted by -0.5 (about 69% of ReLU(K) is zero): the un-rotated denominator stays >= eps.
    rng = np.random.default_rng(10)
    N, d = 400, 32
    q = _rand(rng, N, d)
    k = _rand(rng, N, d) - 0.5
    qp, kp = orc.relu(q), orc.relu(k)
    den = qp @ kp.sum(axis=0) + 1e-6
    assert np.all(den >= 1e-6)
    assert 0.6 < np.mean(kp == 0.0) < 0.75


# --------------------------------------------------------------------------
# Block-causal mode
# --------------------------------------------------------------------------

def _small_blockcausal(rng, grid=(7, 3, 4), d=16, bands=(4, 6, 6), H=2):
    N = grid[0] * grid[1] * grid[2]
    return [_rand(rng, 1, H, N, d) for _ in range(4)], grid, d, bands


@pytest.mark.parametrize("bf", [1, 2, 3])
def test_blockcausal_equals_masked_brute_form(bf):
    rng = np.random.default_rng(11 + bf)
    (q, k, v, g), grid, d, bands = _small_blockcausal(rng)
    O = orc.forward_blockcausal(q, k, v, g, grid, bands, 10000.0, 1e-6, block_frames=bf)
    pos = orc.grid_positions(*grid)
    blk = pos[:, 0] // bf
    visible = blk[None, :] <= blk[:, None]  # token n reads every key of blocks <= its own
    for h in range(q.shape[1]):
        ob = orc.forward_brute(q[0, h], k[0, h], v[0, h], g[0, h], pos, bands, 10000.0, 1e-6, visible)
        assert np.max(np.abs(ob - O[0, h])) <= 1e-11 * np.max(np.abs(ob))


def test_blockcausal_last_block_equals_bidirectional():
    rng = np.random.default_rng(20)
    (q, k, v, g), grid, d, bands = _small_blockcausal(rng)
    Ob, Sb, zb = orc.forward_bidir(q, k, v, g, grid, bands, 10000.0, 1e-6, return_state=True)
    Oc, Sc, zc = orc.forward_blockcausal(q, k, v, g, grid, bands, 10000.0, 1e-6, block_frames=2,
                                         return_state=True)
    assert np.allclose(Sc[:, :, -1], Sb, atol=1e-12)
    assert np.allclose(zc[:, :, -1], zb, atol=1e-12)
    last = orc.grid_positions(*grid)[:, 0] // 2 == Sc.shape[2] - 1
    assert np.allclose(Oc[:, :, last], Ob[:, :, last], rtol=1e-12, atol=1e-14)


def test_blockcausal_one_block_is_bidirectional_and_first_block_is_local():
    rng = np.random.default_rng(21)
    (q, k, v, g), grid, d, bands = _small_blockcausal(rng)
    Ob = orc.forward_bidir(q, k, v, g, grid, bands, 10000.0, 1e-6)
    for bf in (grid[0], grid[0] + 5):
        Oc = orc.forward_blockcausal(q, k, v, g, grid, bands, 10000.0, 1e-6, block_frames=bf)
        assert np.allclose(Oc, Ob, rtol=1e-12, atol=1e-14)
    # Block 0 (2 frames) equals a bidirectional run on those frames alone.
    n0 = 2 * grid[1] * grid[2]
    Oc = orc.forward_blockcausal(q, k, v, g, grid, bands, 10000.0, 1e-6, block_frames=2)
    O0 = orc.forward_bidir(q[:, :, :n0], k[:, :, :n0], v[:, :, :n0], g[:, :, :n0],
                           (2, grid[1], grid[2]), bands, 10000.0, 1e-6)
    assert np.allclose(Oc[:, :, :n0], O0, rtol=1e-12, atol=1e-14)


def test_blockcausal_inclusive_states_are_prefix_sums_of_block_states():
    rng = np.random.default_rng(22)
    (q, k, v, g), grid, d, bands = _small_blockcausal(rng, H=1)
    _, Sc, zc = orc.forward_blockcausal(q, k, v, g, grid, bands, 10000.0, 1e-6, block_frames=3,
                                        return_state=True)
    pos = orc.grid_positions(*grid)
    Sb, zb = orc.block_states(k[0, 0], v[0, 0], pos, bands, 10000.0, 3)
    assert Sb.shape[0] == 3  # 7 frames in blocks of 3: 3, 3, 1
    assert np.allclose(np.cumsum(Sb, axis=0), Sc[0, 0], atol=1e-12)
    assert np.allclose(np.cumsum(zb, axis=0), zc[0, 0], atol=1e-12)


# --------------------------------------------------------------------------
# Planted mistakes: each must be caught by one of the pins above
# --------------------------------------------------------------------------

def _rotated_denominator_forward(q, k, v, g, pos, bands, base, eps):
    qp, kp = orc.relu(q), orc.relu(k)
    qr, kr = orc.rope3d(qp, pos, bands, base), orc.rope3d(kp, pos, bands, base)
    return (qr @ (kr.T @ v)) / ((qr @ kr.sum(0)) + eps)[:, None] * orc.sigmoid(g)


def test_planted_rotated_denominator_is_caught():
    d = 8
    q = np.zeros((2, d)); k = np.zeros((2, d)); q[:, 0] = 1.0; k[:, 0] = 1.0
    v = np.eye(2, d)
    g = np.full((2, d), 50.0)
    pos = orc.grid_positions(2, 1, 1)
    good = orc.forward_positions(q, k, v, g, pos, (2, 2, 4), 10000.0, 1e-6)
    bad = _rotated_denominator_forward(q, k, v, g, pos, (2, 2, 4), 10000.0, 1e-6)
    expect0 = (v[0] + math.cos(1.0) * v[1]) / (2.0 + 1e-6)
    assert np.allclose(good[0], expect0, rtol=1e-13)
    assert not np.allclose(bad[0], expect0, rtol=1e-3)


def test_planted_transposed_state_is_caught_by_brute_form():
    rng = np.random.default_rng(30)
    N, d, bands = 24, 8, (2, 2, 4)
    q, k, v, g = (_rand(rng, N, d) for _ in range(4))
    pos = orc.grid_positions(2, 3, 4)
    S, z = orc.head_state(k, v, pos, bands, 10000.0)
    bad = orc.head_apply(q, g, S.T, z, pos, bands, 10000.0, 1e-6)
    ob = orc.forward_brute(q, k, v, g, pos, bands, 10000.0, 1e-6)
    assert np.max(np.abs(bad - ob)) > 1e-3 * np.max(np.abs(ob))


def test_streaming_cache_restatement_equals_block_causal_form():
    """Algorithm 1 of the block-causal paper, restated: carry (S, z), fold each block's keys and
    values in (RoPE at global frame indices), then apply the block against the carried state.
    This must reproduce the block-causal operator exactly (up to fp64 rounding)."""
    rng = np.random.default_rng(11)
    T, Hh, W, d, bands, bf = 7, 3, 4, 16, (4, 6, 6), 2
    N = T * Hh * W
    q, k, v, g = (rng.standard_normal((1, 1, N, d)) for _ in range(4))
    ref = orc.forward_blockcausal(q, k, v, g, (T, Hh, W), bands, 10000.0, 1e-6, block_frames=bf)[0, 0]
    S, z = np.zeros((d, d)), np.zeros(d)
    out = []
    for t0 in range(0, T, bf):
        t1 = min(T, t0 + bf)
        sl = slice(t0 * Hh * W, t1 * Hh * W)
        pos = orc.grid_positions(t1 - t0, Hh, W)
        pos[:, 0] += t0
        Sb, zb = orc.head_state(k[0, 0, sl], v[0, 0, sl], pos, bands, 10000.0)
        S, z = S + Sb, z + zb
        out.append(orc.head_apply(q[0, 0, sl], g[0, 0, sl], S, z, pos, bands, 10000.0, 1e-6))
    assert np.allclose(np.concatenate(out), ref, rtol=1e-12, atol=1e-14)
    # Positions local to the block (t0 ignored) give a different result: the offset matters.
    pos_local = orc.grid_positions(T - 6, Hh, W)
    sl = slice(6 * Hh * W, N)
    bad = orc.head_apply(q[0, 0, sl], g[0, 0, sl], S, z, pos_local, bands, 10000.0, 1e-6)
    assert not np.allclose(bad, ref[sl], rtol=1e-3)


# ----------------------------------------------------------------- full Eq. (1): write gate, RMSNorm

def _rand_head(rng, N, d):
    return [rng.standard_normal((N, d)) for _ in range(4)]


def test_gated_linear_form_equals_brute_form():
    """beta and RMSNorm in the linear form agree with the pair-wise form (SANA-Video 2.0, Eq. (1))."""
    rng = np.random.default_rng(21)
    T, Hh, W, d, bands = 3, 2, 5, 16, (4, 6, 6)
    pos = orc.grid_positions(T, Hh, W)
    q, k, v, g = _rand_head(rng, T * Hh * W, d)
    beta = rng.uniform(0.0, 1.0, T * Hh * W)
    gamma = 1.0 + 0.1 * rng.standard_normal(d)
    for b_, rms in ((beta, None), (None, (gamma, 1e-6)), (beta, (gamma, 1e-6)), (beta, (None, 0.0))):
        lin = orc.forward_positions(q, k, v, g, pos, bands, 10000.0, 1e-6, beta=b_, rms=rms)
        bru = orc.forward_brute(q, k, v, g, pos, bands, 10000.0, 1e-6, beta=b_, rms=rms)
        assert np.allclose(lin, bru, rtol=1e-11, atol=1e-13)


def test_write_gate_two_token_closed_form():
    """Two tokens at one position, q = k_0 = k_1 = e_0, beta = (1, 0), g = 0: the gate removes
    token 1 from the numerator only, so o = v_0 / (2 + eps) / 2.  (Gating the denominator too,
    a plausible misreading, would give v_0 / (1 + eps) / 2.)"""
    d, bands = 8, (2, 2, 4)
    e0 = np.zeros(d); e0[0] = 1.0
    q = np.array([e0, e0]); k = np.array([e0, e0])
    v = np.array([[1.0, -2.0, 3.0, 0.5, 0.0, 1.0, 2.0, -1.0], [5.0, 5.0, 5.0, 5.0, 5.0, 5.0, 5.0, 5.0]])
    g = np.zeros((2, d))
    pos = np.array([[1, 2, 3], [1, 2, 3]])
    out = orc.forward_positions(q, k, v, g, pos, bands, 10000.0, 1e-6, beta=np.array([1.0, 0.0]))
    assert np.allclose(out[0], v[0] / (2.0 + 1e-6) / 2.0, rtol=1e-13)
    assert not np.allclose(out[0], v[0] / (1.0 + 1e-6) / 2.0, rtol=1e-3)
    # beta = 1 everywhere is the plain operator
    plain = orc.forward_positions(q, k, v, g, pos, bands, 10000.0, 1e-6)
    ones = orc.forward_positions(q, k, v, g, pos, bands, 10000.0, 1e-6, beta=np.ones(2))
    assert np.array_equal(plain, ones)


def test_rms_norm_single_token_closed_form():
    """N = 1: y = a v with a = s / (s + eps); with norm_eps = 0 the factor a cancels and
    RMSNorm(y) = v / sqrt(mean(v^2)) * gamma.  v = (3, 4, 0, ...) over d = 8 has mean(v^2) = 25/8."""
    d, bands = 8, (2, 2, 4)
    q = np.zeros((1, d)); q[0, 0] = 2.0
    k = np.zeros((1, d)); k[0, 0] = 3.0
    v = np.zeros((1, d)); v[0, 0], v[0, 1] = 3.0, 4.0
    g = np.zeros((1, d))
    gamma = np.array([1.0, 2.0, 1.0, 1.0, 1.0, 1.0, 1.0, 1.0])
    out = orc.forward_positions(q, k, v, g, np.array([[4, 0, 7]]), bands, 10000.0, 1e-6, rms=(gamma, 0.0))
    expect = np.zeros(d)
    expect[0] = 3.0 / np.sqrt(25.0 / 8.0) * 0.5
    expect[1] = 8.0 / np.sqrt(25.0 / 8.0) * 0.5
    assert np.allclose(out[0], expect, rtol=1e-12, atol=1e-15)


def test_rms_norm_invariances_and_placement():
    rng = np.random.default_rng(23)
    T, Hh, W, d, bands = 2, 3, 4, 16, (4, 6, 6)
    pos = orc.grid_positions(T, Hh, W)
    q, k, v, g = _rand_head(rng, T * Hh * W, d)
    rms = (None, 0.0)
    base = orc.forward_positions(q, k, v, g, pos, bands, 10000.0, 1e-6, rms=rms)
    # scale of V (and of the write gate) drops out of a normalised row
    assert np.allclose(orc.forward_positions(q, k, 7.5 * v, g, pos, bands, 10000.0, 1e-6, rms=rms), base,
                       rtol=1e-12)
    assert np.allclose(orc.forward_positions(q, k, v, g, pos, bands, 10000.0, 1e-6, beta=np.full(len(q), 0.3),
                                             rms=rms), base, rtol=1e-12)
    # every row of O / sigmoid(G) has unit RMS (gamma = 1, norm_eps = 0)
    y = base / orc.sigmoid(g)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, rtol=1e-12)
    # placement: normalising after the gate (the other rendering of Eq. (1)) is a different result
    plain = orc.forward_positions(q, k, v, g, pos, bands, 10000.0, 1e-6)
    after = orc.rms_norm(plain, None, 0.0)
    assert not np.allclose(after, base, rtol=1e-3)


# ----------------------------------------------------------------- token-causal form

def test_tokencausal_linear_form_equals_masked_brute_form():
    rng = np.random.default_rng(31)
    for T, Hh, W, d, bands in ((3, 2, 5, 16, (4, 6, 6)), (2, 3, 4, 8, (2, 2, 4))):
        N = T * Hh * W
        pos = orc.grid_positions(T, Hh, W)
        q, k, v, g = (rng.standard_normal((N, d)) for _ in range(4))
        lin = orc.tokencausal_rows(q, k, v, g, pos, bands, 10000.0, 1e-6)
        mask = np.tril(np.ones((N, N), dtype=bool))
        bru = orc.forward_brute(q, k, v, g, pos, bands, 10000.0, 1e-6, visible=mask)
        assert np.allclose(lin, bru, rtol=1e-11, atol=1e-13)
        # sampled rows agree with the full evaluation
        rows = [0, 5, N - 1, 13]
        assert np.allclose(orc.tokencausal_rows(q, k, v, g, pos, bands, 10000.0, 1e-6, rows=rows),
                           lin[rows], rtol=1e-12)


def test_tokencausal_first_last_and_causality():
    rng = np.random.default_rng(37)
    T, Hh, W, d, bands = 2, 3, 5, 16, (4, 6, 6)
    N = T * Hh * W
    Q, K, V, G = (rng.standard_normal((1, 1, N, d)) for _ in range(4))
    O = orc.forward_tokencausal(Q, K, V, G, (T, Hh, W), bands)[0, 0]
    bid = orc.forward_bidir(Q, K, V, G, (T, Hh, W), bands)[0, 0]
    # the last token sees every token: bidirectional output
    assert np.allclose(O[-1], bid[-1], rtol=1e-12)
    # the first token sees only itself: single-token closed form (same position: rotation cancels)
    qp, kp = np.maximum(Q[0, 0, 0], 0), np.maximum(K[0, 0, 0], 0)
    s = qp @ kp
    assert np.allclose(O[0], s / (s + 1e-6) * V[0, 0, 0] / (1 + np.exp(-G[0, 0, 0])), rtol=1e-10)
    # changing token j changes no output before j
    j = 11
    K2, V2 = K.copy(), V.copy()
    K2[0, 0, j] += 1.0
    V2[0, 0, j] -= 2.0
    O2 = orc.forward_tokencausal(Q, K2, V2, G, (T, Hh, W), bands)[0, 0]
    assert np.array_equal(O2[:j], O[:j])
    assert not np.allclose(O2[j:], O[j:])


# ----------------------------------------------------------------- gradients

def _loss(q, k, v, g, do, pos, bands):
    return float(np.sum(orc.forward_positions(q, k, v, g, pos, bands, 10000.0, 1e-6) * do))


def test_backward_matches_central_differences():
    """The oracle's gradients against central finite differences of the forward oracle (fp64):
    d/dx sum(O * dO) for every input element of a small head."""
    rng = np.random.default_rng(41)
    T, Hh, W, d, bands = 2, 2, 3, 8, (2, 2, 4)
    N = T * Hh * W
    pos = orc.grid_positions(T, Hh, W)
    q, k, v, g, do = (rng.standard_normal((N, d)) for _ in range(5))
    # keep every entry away from the ReLU kink so the differences see a smooth function
    for x in (q, k):
        x[np.abs(x) < 0.05] = 0.3
    grads = orc.head_backward(q, k, v, g, do, pos, bands, 10000.0, 1e-6)
    h = 1e-6
    for which, grad in enumerate(grads):
        args = [q, k, v, g]
        fd = np.empty_like(args[which])
        for idx in np.ndindex(*fd.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd[idx] = (_loss(*plus, do, pos, bands) - _loss(*minus, do, pos, bands)) / (2 * h)
        assert np.allclose(grad, fd, rtol=1e-6, atol=1e-7), which


def test_rope_transpose_is_the_inverse_rotation():
    rng = np.random.default_rng(43)
    pos = orc.grid_positions(3, 4, 5)
    x = rng.standard_normal((len(pos), 16))
    bands = (4, 6, 6)
    assert np.allclose(orc.rope3d_transpose(orc.rope3d(x, pos, bands, 10000.0), pos, bands, 10000.0), x,
                       rtol=1e-13, atol=1e-14)
    y = rng.standard_normal(x.shape)
    # <R x, y> = <x, R^T y> row by row
    assert np.allclose(np.sum(orc.rope3d(x, pos, bands, 10000.0) * y, axis=1),
                       np.sum(x * orc.rope3d_transpose(y, pos, bands, 10000.0), axis=1), rtol=1e-12)


def test_multihead_wrappers_take_each_head_separately():
    # Two heads (B = 1, H = 2) through the [B, H, N, d] wrappers: each head's result is that of
    # the masked brute form (token-causal) or the central differences pinned above (gradients)
    # on that head alone, so a mix-up of heads or of the B/H order fails here.
    rng = np.random.default_rng(47)
    T, Hh, W, d, bands = 2, 2, 3, 8, (2, 2, 4)
    N = T * Hh * W
    pos = orc.grid_positions(T, Hh, W)
    Q, K, V, G, dO = (rng.standard_normal((1, 2, N, d)) for _ in range(5))
    Q[:, 1] *= 3.0  # make the heads differ in scale too
    O = orc.forward_tokencausal(Q, K, V, G, (T, Hh, W), bands)
    mask = np.tril(np.ones((N, N), dtype=bool))
    for h in range(2):
        bru = orc.forward_brute(Q[0, h], K[0, h], V[0, h], G[0, h], pos, bands, 10000.0, 1e-6, visible=mask)
        assert np.allclose(O[0, h], bru, rtol=1e-11, atol=1e-13)
    grads = orc.backward_bidir(Q, K, V, G, dO, (T, Hh, W), bands)
    for h in range(2):
        args = [Q[0, h].copy(), K[0, h].copy(), V[0, h].copy(), G[0, h].copy()]
        for x in args[:2]:
            x[np.abs(x) < 0.05] = 0.3
        Qh, Kh = Q.copy(), K.copy()
        Qh[0, h], Kh[0, h] = args[0], args[1]
        gh = orc.backward_bidir(Qh, Kh, V, G, dO, (T, Hh, W), bands)
        fd = _fd_grads(lambda a: _loss(*a, dO[0, h], pos, bands), args)
        for which in range(4):
            assert np.allclose(gh[which][0, h], fd[which], rtol=1e-6, atol=1e-7), (h, which)
    assert grads[0].shape == Q.shape


def _fd_grads(loss, args, h=1e-6):
    """Central differences of loss(args) with respect to every element of every array in args."""
    out = []
    for which in range(len(args)):
        fd = np.empty_like(args[which])
        for idx in np.ndindex(*fd.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd[idx] = (loss(plus) - loss(minus)) / (2 * h)
        out.append(fd)
    return out


@pytest.mark.parametrize("block_frames,use_beta,use_rms", [
    (1, False, False), (2, False, False), (0, True, False), (0, False, True), (2, True, True)])
def test_gated_blockcausal_backward_matches_central_differences(block_frames, use_beta, use_rms):
    """Gradients of the full form (block-causal states, write gate beta, RMSNorm with gamma) against
    central differences of the forward oracle: d/dx sum(O * dO) for every element of q, k, v, g,
    beta and gamma."""
    rng = np.random.default_rng(53 + 7 * block_frames + 2 * use_beta + use_rms)
    T, Hh, W, d, bands = 3, 2, 2, 8, (2, 2, 4)
    N = T * Hh * W
    pos = orc.grid_positions(T, Hh, W)
    q, k, v, g, do = (rng.standard_normal((N, d)) for _ in range(5))
    for x in (q, k):
        x[np.abs(x) < 0.05] = 0.3
    beta = rng.uniform(0.2, 1.5, N) if use_beta else None
    gamma = rng.uniform(0.5, 1.5, d) if use_rms else None
    rms = (gamma, 1e-3) if use_rms else None

    def fwd(q_, k_, v_, g_, beta_, gamma_):
        r = (gamma_, 1e-3) if use_rms else None
        shape = (1, 1, N, d)
        b4 = None if beta_ is None else beta_.reshape(1, 1, N)
        if block_frames > 0:
            return orc.forward_blockcausal(q_.reshape(shape), k_.reshape(shape), v_.reshape(shape),
                                           g_.reshape(shape), (T, Hh, W), bands, block_frames=block_frames,
                                           beta=b4, rms=r)[0, 0]
        return orc.forward_positions(q_, k_, v_, g_, pos, bands, 10000.0, 1e-6, beta=beta_, rms=r)

    args = [q, k, v, g] + ([beta] if use_beta else []) + ([gamma] if use_rms else [])

    def loss(a):
        it = iter(a[4:])
        b_ = next(it) if use_beta else None
        gm = next(it) if use_rms else None
        return float(np.sum(fwd(a[0], a[1], a[2], a[3], b_, gm) * do))

    dq, dk, dv, dg, dbeta, dgamma = orc.head_backward_gated(q, k, v, g, do, pos, bands, 10000.0, 1e-6,
                                                            block_frames, beta, rms)
    got = [dq, dk, dv, dg] + ([dbeta] if use_beta else []) + ([dgamma] if use_rms else [])
    fd = _fd_grads(loss, args)
    for i, (a, b) in enumerate(zip(got, fd)):
        assert np.allclose(a, b, rtol=1e-6, atol=2e-7), i
    assert (dbeta is None) == (not use_beta) and (dgamma is None) == (not use_rms)


def test_gated_backward_reduces_to_the_plain_bidirectional_gradients():
    rng = np.random.default_rng(59)
    T, Hh, W, d, bands = 2, 3, 4, 16, (4, 6, 6)
    N = T * Hh * W
    pos = orc.grid_positions(T, Hh, W)
    q, k, v, g, do = (rng.standard_normal((N, d)) for _ in range(5))
    plain = orc.head_backward(q, k, v, g, do, pos, bands, 10000.0, 1e-6)
    full = orc.head_backward_gated(q, k, v, g, do, pos, bands, 10000.0, 1e-6)
    for a, b in zip(plain, full[:4]):
        assert np.allclose(a, b, rtol=1e-12, atol=1e-14)
    # one block covering every frame is the bidirectional form
    one = orc.head_backward_gated(q, k, v, g, do, pos, bands, 10000.0, 1e-6, block_frames=T)
    for a, b in zip(plain, one[:4]):
        assert np.allclose(a, b, rtol=1e-12, atol=1e-14)
    # beta = 1 gives the un-gated gradients and dbeta = phi(k) . (dS v)
    ones = orc.head_backward_gated(q, k, v, g, do, pos, bands, 10000.0, 1e-6, beta=np.ones(N))
    for a, b in zip(plain, ones[:4]):
        assert np.allclose(a, b, rtol=1e-12, atol=1e-14)
