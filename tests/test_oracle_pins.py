"""Pins of the float64 oracle against brute force, closed forms, library
routines and invariants (no GPU).  Each pin is chosen so that a plausible
mistake in the oracle (a dropped term, a wrong sign or index, a transposed
operand, RoPE in the denominator, a wrong axis split) fails at least one."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import sana_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def rand(*shape):
    return rng.standard_normal(shape)


def rel(a, b):
    return orc.max_rel_err(a, b)


# ---------------------------------------------------------------- RoPE (P3)

def test_rope_angles_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "rope_angles_tiny.json")))
    ang = orc.rope_angles(*g["grid"], *g["split"])
    for e in g["entries"]:
        np.testing.assert_allclose(ang[e["token"]], e["angles"], rtol=1e-12, atol=1e-15)
        T, H, W = g["grid"]
        t, h, w = orc.token_grid(T, H, W)
        assert [t[e["token"]], h[e["token"]], w[e["token"]]] == e["thw"]


def test_rope_single_pair_closed_form():
    # D = 2: (x, y) rotated by a -> (x cos a - y sin a, x sin a + y cos a)
    x, y, a = 0.7, -1.3, 0.9
    out = orc.apply_rope(np.array([[x, y]]), np.array([[a]]))
    exp = [x * math.cos(a) - y * math.sin(a), x * math.sin(a) + y * math.cos(a)]
    np.testing.assert_allclose(out[0], exp, rtol=1e-15)


def test_rope_preserves_pair_norms():
    x = rand(3, 40, 16)
    ang = rand(40, 8) * 5
    r = orc.apply_rope(x, ang)
    np.testing.assert_allclose(np.hypot(r[..., 0::2], r[..., 1::2]),
                               np.hypot(x[..., 0::2], x[..., 1::2]), rtol=1e-13)


def test_rope_offset_absolute_frames():
    a0 = orc.rope_angles(3, 2, 2, 2, 1, 1, t_offset=5)
    a1 = orc.rope_angles(8, 2, 2, 2, 1, 1)[5 * 4:]
    np.testing.assert_allclose(a0, a1, rtol=0, atol=0)


# ------------------------------------------------- bidirectional linear attention

def _lin_inputs(B, N, heads, D, gate=True):
    C = heads * D
    return (rand(B, N, C), rand(B, N, C), rand(B, N, C),
            rand(B, N, C) if gate else None)


@pytest.mark.parametrize("grid,split,heads,D", [
    ((2, 4, 4), (2, 3, 3), 2, 16),      # the tiny workload
    ((3, 5, 7), (2, 3, 3), 1, 16),      # N = 105, ragged against any tile size
    ((5, 7, 8), (1, 1, 2), 3, 8),       # N = 280
    ((1, 1, 1), (0, 0, 4), 2, 8),       # a single token
])
def test_factorised_equals_bruteforce(grid, split, heads, D):
    """P1: the associativity of the linear form (sec. 3.2 pseudocode)."""
    N = grid[0] * grid[1] * grid[2]
    q, k, v, g = _lin_inputs(2, N, heads, D)
    y, S, z = orc.linattn_bidirectional(q, k, v, grid, split, heads, gate=g)
    yb = orc.linattn_bruteforce(q, k, v, grid, split, heads, gate=g)
    assert rel(y, yb) < 1e-12


def test_linear_attention_d2_worked_example():
    """A hand-worked D = 2 example: one head, tokens at w = 0 and w = 1
    (angle 0 and 1 rad).  q0=(1,0), q1=(.5,2), k0=(1,1), k1=(2,-1),
    v0=(1,2), v1=(3,-1).  phi(k1) = (2,0), so
    S = [[1 + 6 cos1, 2 - 2 cos1], [1 + 6 sin1, 2 - 2 sin1]], z = (3, 1).
    Token 0: numerator = row 0 of S, denominator 3.
    Token 1: RoPE(phi q1) = (.5 cos1 - 2 sin1, .5 sin1 + 2 cos1), denominator
    .5*3 + 2*1 = 3.5."""
    c, s = math.cos(1.0), math.sin(1.0)
    S = np.array([[1 + 6 * c, 2 - 2 * c], [1 + 6 * s, 2 - 2 * s]])
    eps = orc.EPS
    o0 = S[0] / (3 + eps)
    qr = np.array([0.5 * c - 2 * s, 0.5 * s + 2 * c])
    o1 = (qr @ S) / (3.5 + eps)
    q = np.array([[[1, 0], [0.5, 2]]], float)
    k = np.array([[[1, 1], [2, -1]]], float)
    v = np.array([[[1, 2], [3, -1]]], float)
    y, S_o, z_o = orc.linattn_bidirectional(q, k, v, (1, 1, 2), (0, 0, 1), 1)
    np.testing.assert_allclose(S_o[0, 0], S, rtol=1e-14)
    np.testing.assert_allclose(z_o[0, 0], [3, 1], rtol=1e-15)
    np.testing.assert_allclose(y[0], np.stack([o0, o1]), rtol=1e-13)


def test_positions_zero_reduce_to_plain_relu_linear_attention():
    """P3/P4: with every angle 0 RoPE is the identity; with V = c the output
    is c * d / (d + eps) with d = phi(Q) . z."""
    N, D = 24, 8
    q, k, _, _ = _lin_inputs(1, N, 1, D, gate=False)
    # a grid of a single position on every axis used: all angles zero
    ang0 = np.zeros((N, D // 2))
    S, z = orc.linattn_state(k, np.ones((1, N, D)) * 1.5, ang0, 1)
    y = orc.linattn_apply(q, S, z, ang0, 1)
    d = np.maximum(q, 0) @ np.maximum(k, 0)[0].sum(0)
    np.testing.assert_allclose(y[0], (1.5 * d / (d + orc.EPS))[0][:, None] * np.ones(D),
                               rtol=1e-12)
    # and the general no-RoPE case equals plain ReLU linear attention
    v = rand(1, N, D)
    S, z = orc.linattn_state(k, v, ang0, 1)
    y = orc.linattn_apply(q, S, z, ang0, 1)
    qp, kp = np.maximum(q[0], 0), np.maximum(k[0], 0)
    plain = (qp @ kp.T @ v[0]) / ((qp @ kp.T).sum(1, keepdims=True) + orc.EPS)
    assert rel(y[0], plain) < 1e-12


def test_denominator_carries_no_rope():
    """The denominator is phi(Q).sum phi(K) without rotation: with V = 1 and
    angles != 0 the output differs from the rotated-denominator variant."""
    grid, split = (2, 3, 3), (1, 1, 2)
    N, D = 18, 8
    q, k, _, _ = _lin_inputs(1, N, 1, D, gate=False)
    ang = orc.rope_angles(*grid, *split)
    S, z = orc.linattn_state(k, rand(1, N, D), ang, 1)
    qp = np.maximum(q[0], 0)
    den_norope = qp @ np.maximum(k[0], 0).sum(0)
    y = orc.linattn_apply(q, S, z, ang, 1)
    num = orc.apply_rope(qp, ang) @ S[0, 0]
    np.testing.assert_allclose(y[0], num / (den_norope[:, None] + orc.EPS), rtol=1e-12)


def test_relative_position_shift_invariance():
    """P3: shifting every frame index leaves the bidirectional output unchanged."""
    grid, split = (3, 3, 4), (2, 1, 1)
    N = 36
    q, k, v, g = _lin_inputs(1, N, 2, 8)
    y0, _, _ = orc.linattn_bidirectional(q, k, v, grid, split, 2, gate=g)
    y1, _, _ = orc.linattn_bidirectional(q, k, v, grid, split, 2, gate=g, t_offset=17)
    assert rel(y1, y0) < 1e-12


def test_gate_limits():
    """P7: gate logits -> +inf give the ungated output, -> -inf give 0."""
    grid, split = (2, 2, 2), (1, 1, 2)
    q, k, v, _ = _lin_inputs(1, 8, 1, 8, gate=False)
    y, _, _ = orc.linattn_bidirectional(q, k, v, grid, split, 1)
    yp, _, _ = orc.linattn_bidirectional(q, k, v, grid, split, 1, gate=np.full(q.shape, 60.0))
    ym, _, _ = orc.linattn_bidirectional(q, k, v, grid, split, 1, gate=np.full(q.shape, -60.0))
    assert rel(yp, y) < 1e-15
    assert np.max(np.abs(ym)) <= 1e-25 * np.max(np.abs(y))


def test_state_size_independent_of_n():
    """P8: the state is D x D plus D per head whatever N is (sec. 3.4 table)."""
    for T in (1, 4, 9):
        grid = (T, 2, 2)
        N = 4 * T
        _, k, v, _ = _lin_inputs(1, N, 3, 8, gate=False)
        S, z = orc.linattn_state(k, v, orc.rope_angles(*grid, 1, 1, 2), 3)
        assert S.shape == (1, 3, 8, 8) and z.shape == (1, 3, 8)


# ------------------------------------------------------------- block-causal (P2)

def _frame_mask(grid, chunk_sizes):
    T, H, W = grid
    frame_chunk = np.concatenate([[c] * f for c, f in enumerate(chunk_sizes)])
    tok_chunk = np.repeat(frame_chunk, H * W)
    return tok_chunk[None, :] <= tok_chunk[:, None]


def _run_chunks(q, k, v, g, grid, split, heads, chunk_sizes, S0=None, z0=None, eps=orc.EPS):
    T, H, W = grid
    B, N, C = q.shape
    D = C // heads
    S = np.zeros((B, heads, D, D)) if S0 is None else S0
    z = np.zeros((B, heads, D)) if z0 is None else z0
    ys, states = [], []
    t0 = 0
    for f in chunk_sizes:
        sl = slice(t0 * H * W, (t0 + f) * H * W)
        y, S, z = orc.linattn_block_causal_step(
            q[:, sl], k[:, sl], v[:, sl], (f, H, W), t0, split, heads, S, z,
            gate=None if g is None else g[:, sl], eps=eps)
        ys.append(y)
        states.append((S.copy(), z.copy()))
        t0 += f
    return np.concatenate(ys, axis=1), states


@pytest.mark.parametrize("chunks", [[1] * 6, [2, 2, 2], [3, 3], [5, 1], [1, 2, 3], [6]])
def test_chunked_equals_masked_bruteforce(chunks):
    grid, split, heads = (6, 2, 3), (2, 1, 1), 2
    N = 36
    q, k, v, g = _lin_inputs(1, N, heads, 8)
    y, _ = _run_chunks(q, k, v, g, grid, split, heads, chunks)
    yb = orc.linattn_bruteforce(q, k, v, grid, split, heads, gate=g,
                                mask=_frame_mask(grid, chunks))
    assert rel(y, yb) < 1e-12


@pytest.mark.parametrize("frames", [1, 2, 3, 4, 7, 9])
def test_block_sequence_equals_masked_bruteforce(frames):
    """A whole sequence in blocks of `frames` frames (7 = 3 + 3 + 1 for
    frames=3, one block when frames >= 7): brute force with chunk(j) <= chunk(i)."""
    grid, split, heads = (7, 2, 3), (2, 1, 1), 2
    T = grid[0]
    N = T * 6
    q, k, v, g = _lin_inputs(1, N, heads, 8)
    S0, z0 = np.zeros((1, heads, 8, 8)), np.zeros((1, heads, 8))
    y, S, z = orc.linattn_block_causal_sequence(q, k, v, grid, frames, 0, split, heads, S0, z0,
                                                gate=g)
    sizes = [min(frames, T - t) for t in range(0, T, frames)]
    yb = orc.linattn_bruteforce(q, k, v, grid, split, heads, gate=g, mask=_frame_mask(grid, sizes))
    assert rel(y, yb) < 1e-12
    _, S_bi, z_bi = orc.linattn_bidirectional(q, k, v, grid, split, heads, gate=g)
    assert rel(S, S_bi) < 1e-13 and rel(z, z_bi) < 1e-13


def test_block_sequence_resumes_from_a_carried_state():
    """Frames [0, 4) then [4, 7) from the carried state (absolute frames from
    t_offset = 4) equal the whole sequence; without commit the state is kept."""
    grid, split, heads = (7, 2, 3), (2, 1, 1), 2
    hw = 6
    q, k, v, g = _lin_inputs(2, 7 * hw, heads, 8)
    S0, z0 = np.zeros((2, heads, 8, 8)), np.zeros((2, heads, 8))
    y_all, S_all, z_all = orc.linattn_block_causal_sequence(q, k, v, grid, 2, 0, split, heads,
                                                            S0, z0, gate=g)
    a, r = slice(0, 4 * hw), slice(4 * hw, 7 * hw)
    y_a, S_a, z_a = orc.linattn_block_causal_sequence(q[:, a], k[:, a], v[:, a], (4, 2, 3), 2, 0,
                                                      split, heads, S0, z0, gate=g[:, a])
    y_r, S_r, z_r = orc.linattn_block_causal_sequence(q[:, r], k[:, r], v[:, r], (3, 2, 3), 2, 4,
                                                      split, heads, S_a, z_a, gate=g[:, r])
    assert rel(np.concatenate([y_a, y_r], axis=1), y_all) < 1e-13
    assert rel(S_r, S_all) < 1e-13 and rel(z_r, z_all) < 1e-13
    y_n, S_n, z_n = orc.linattn_block_causal_sequence(q[:, r], k[:, r], v[:, r], (3, 2, 3), 2, 4,
                                                      split, heads, S_a, z_a, gate=g[:, r],
                                                      commit=False)
    assert rel(y_n, y_r) == 0 and np.array_equal(S_n, S_a) and np.array_equal(z_n, z_a)


@pytest.mark.parametrize("gated,B,grid,split,heads,D", [
    (True, 1, (2, 3, 4), (2, 1, 1), 2, 8),
    (False, 2, (3, 5, 7), (2, 3, 3), 1, 16),   # N = 105
    (True, 2, (1, 1, 1), (0, 0, 4), 2, 8),     # a single token
])
def test_backward_matches_central_finite_differences(gated, B, grid, split, heads, D):
    """<dL/dx, u> for L = sum(dY * Y) against (L(x + h u) - L(x - h u)) / 2h,
    for a random direction u in each of Q, K, V (and G)."""
    N = grid[0] * grid[1] * grid[2]
    C = heads * D
    q, k, v, dy = (rand(B, N, C) for _ in range(4))
    g = rand(B, N, C) if gated else None
    grads = orc.linattn_backward(q, k, v, grid, split, heads, dy, gate=g)

    def loss(qq, kk, vv, gg):
        return (orc.linattn_bidirectional(qq, kk, vv, grid, split, heads, gate=gg)[0] * dy).sum()

    h = 1e-6
    names = ["q", "k", "v"] + (["g"] if gated else [])
    for name, grad in zip(names, grads):
        u = rand(B, N, C)
        args = dict(qq=q, kk=k, vv=v, gg=g)
        key = name * 2
        x = args[key]
        args[key] = x + h * u
        lp = loss(**args)
        args[key] = x - h * u
        lm = loss(**args)
        fd = (lp - lm) / (2 * h)
        assert abs(fd - (grad * u).sum()) <= 1e-7 * max(1.0, abs(fd)), (name, fd, (grad * u).sum())
    assert grads[3] is None or gated


def test_backward_of_v_is_linear_and_ignores_the_gate_scale_of_q():
    """dV = K'^T-weighted sum of dnum (the layer is linear in V): scaling dY
    scales every gradient; dV equals the finite difference exactly for a
    linear layer even with a large step."""
    grid, split, heads, D = (2, 2, 3), (1, 1, 2), 1, 8
    N = 12
    q, k, v, dy = (rand(1, N, D) for _ in range(4))
    g1 = orc.linattn_backward(q, k, v, grid, split, heads, dy)
    g2 = orc.linattn_backward(q, k, v, grid, split, heads, 3.0 * dy)
    for a, b in zip(g1[:3], g2[:3]):
        assert rel(3.0 * a, b) < 1e-14
    u = rand(1, N, D)
    y0 = orc.linattn_bidirectional(q, k, v, grid, split, heads)[0]
    y1 = orc.linattn_bidirectional(q, k, v + 10.0 * u, grid, split, heads)[0]
    assert abs(((y1 - y0) * dy).sum() / 10.0 - (g1[2] * u).sum()) < 1e-10


def test_token_recurrence_equals_prefix_recomputation():
    """Chunk size 1 token: the sec. 3.4 recurrence = brute force with j <= i."""
    grid, split, heads = (2, 3, 4), (2, 1, 1), 2
    N = 24
    q, k, v, _ = _lin_inputs(1, N, heads, 8, gate=False)
    y = orc.linattn_token_recurrence(q, k, v, grid, split, heads)
    mask = np.tril(np.ones((N, N), bool))
    yb = orc.linattn_bruteforce(q, k, v, grid, split, heads, mask=mask)
    assert rel(y, yb) < 1e-12


def test_state_independent_of_chunking_and_full_chunk_is_bidirectional():
    grid, split, heads = (6, 2, 2), (2, 1, 1), 2
    q, k, v, g = _lin_inputs(2, 24, heads, 8)
    _, st_a = _run_chunks(q, k, v, g, grid, split, heads, [1, 2, 3])
    _, st_b = _run_chunks(q, k, v, g, grid, split, heads, [3, 3])
    _, st_c = _run_chunks(q, k, v, g, grid, split, heads, [6])
    # state after the first 3 frames
    assert rel(st_a[1][0], st_b[0][0]) < 1e-13 and rel(st_a[1][1], st_b[0][1]) < 1e-13
    for st in (st_a[-1], st_b[-1]):
        assert rel(st[0], st_c[-1][0]) < 1e-13 and rel(st[1], st_c[-1][1]) < 1e-13
    y_full, _ = _run_chunks(q, k, v, g, grid, split, heads, [6])
    y_bi, S, z = orc.linattn_bidirectional(q, k, v, grid, split, heads, gate=g)
    assert rel(y_full, y_bi) < 1e-13
    assert rel(st_c[-1][0], S) < 1e-13 and rel(st_c[-1][1], z) < 1e-13


def test_commit_flag_and_state_save_restore():
    grid, split, heads = (4, 2, 2), (2, 1, 1), 1
    q, k, v, _ = _lin_inputs(1, 16, heads, 8, gate=False)
    H, W = 2, 2
    S0 = np.zeros((1, 1, 8, 8))
    z0 = np.zeros((1, 1, 8))
    y1, S1, z1 = orc.linattn_block_causal_step(q[:, :8], k[:, :8], v[:, :8], (2, H, W), 0,
                                               split, heads, S0, z0)
    # a non-committing step leaves the state untouched but sees itself
    y_nc, S_nc, z_nc = orc.linattn_block_causal_step(q[:, 8:], k[:, 8:], v[:, 8:], (2, H, W), 2,
                                                     split, heads, S1, z1, commit=False)
    assert np.array_equal(S_nc, S1) and np.array_equal(z_nc, z1)
    # save / restore through a byte round trip is exact
    S_r = np.frombuffer(S1.tobytes()).reshape(S1.shape)
    z_r = np.frombuffer(z1.tobytes()).reshape(z1.shape)
    y2, _, _ = orc.linattn_block_causal_step(q[:, 8:], k[:, 8:], v[:, 8:], (2, H, W), 2,
                                             split, heads, S_r, z_r)
    assert np.array_equal(y2, y_nc)


# ------------------------------------------------------------------ anchor (P5)

def test_anchor_equals_naive_softmax_and_library_sdpa():
    N, D, heads = 40, 8, 2
    q, k, v = rand(1, N, heads * D) * 0.3, rand(1, N, heads * D) * 0.3, rand(1, N, heads * D)
    y = orc.softmax_anchor(q, k, v, None, None, heads, use_rope=False)
    for h in range(heads):
        sl = slice(h * D, (h + 1) * D)
        yn = orc.softmax_naive(q[0, :, sl], k[0, :, sl], v[0, :, sl], D ** -0.5)
        assert rel(y[0, :, sl], yn) < 1e-13
        ys = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[0, :, sl])[None], torch.from_numpy(k[0, :, sl])[None],
            torch.from_numpy(v[0, :, sl])[None]).numpy()[0]
        assert rel(y[0, :, sl], ys) < 1e-12


def test_anchor_with_rope_equals_sdpa_on_rotated_inputs():
    grid, split, heads, D = (2, 3, 4), (1, 1, 2), 2, 8
    N = 24
    q, k, v = rand(1, N, heads * D), rand(1, N, heads * D), rand(1, N, heads * D)
    g = rand(1, N, heads * D)
    y = orc.softmax_anchor(q, k, v, grid, split, heads, gate=g)
    ang = orc.rope_angles(*grid, *split)
    for h in range(heads):
        sl = slice(h * D, (h + 1) * D)
        qr = torch.from_numpy(orc.apply_rope(q[0, :, sl], ang))[None]
        kr = torch.from_numpy(orc.apply_rope(k[0, :, sl], ang))[None]
        ys = torch.nn.functional.scaled_dot_product_attention(
            qr, kr, torch.from_numpy(v[0, :, sl])[None]).numpy()[0]
        assert rel(y[0, :, sl], ys / (1 + np.exp(-g[0, :, sl]))) < 1e-12
    # sampled rows equal the full evaluation
    rows = np.array([0, 5, 23])
    assert rel(orc.softmax_anchor(q, k, v, grid, split, heads, gate=g, rows=rows),
               y[:, rows]) < 1e-15


def test_anchor_special_cases():
    grid, split, heads, D = (1, 2, 5), (0, 2, 2), 1, 8
    N = 10
    q, k = rand(1, N, D), rand(1, N, D)
    v = np.full((1, N, D), 2.5)
    np.testing.assert_allclose(orc.softmax_anchor(q, k, v, grid, split, heads), v, rtol=1e-14)
    # a single key: every query returns that key's value
    y1 = orc.softmax_anchor(q[:, :1], k[:, :1], rand(1, 1, D), (1, 1, 1), split, heads)
    assert y1.shape == (1, 1, D)
    # a constant added to all logits of a row changes nothing (K + c shifts each
    # row of Q K^T by q_i . c when RoPE is off)
    v = rand(1, N, D)
    y = orc.softmax_anchor(q, k, v, None, None, heads, use_rope=False)
    y2 = orc.softmax_anchor(q, k + rand(1, 1, D), v, None, None, heads, use_rope=False)
    assert rel(y2, y) < 1e-12
    # relative RoPE: a frame shift leaves the anchor unchanged
    grid2 = (3, 2, 2)
    q, k, v = rand(1, 12, D), rand(1, 12, D), rand(1, 12, D)
    a = orc.softmax_anchor(q, k, v, grid2, (2, 1, 1), 1)
    b = orc.softmax_anchor(q, k, v, grid2, (2, 1, 1), 1, t_offset=11)
    assert rel(a, b) < 1e-12


# ------------------------------------------- block-sparse anchor (reading)

def _sparse_inputs(N, heads, D, seed_scale=1.0):
    return (rand(1, N, heads * D) * seed_scale, rand(1, N, heads * D) * seed_scale,
            rand(1, N, heads * D), rand(1, N, heads * D))


def test_block_scores_are_mean_logits_of_each_block_pair():
    """q_bar . k_bar = mean over the block pair of the full logit matrix
    (bilinearity), including a ragged last block and tile (N = 600)."""
    grid, split, heads, D = (2, 15, 20), (2, 1, 1), 2, 8
    N = 600
    q, k, _, _ = _sparse_inputs(N, heads, D)
    sc = orc.anchor_block_scores(q, k, grid, split, heads)
    ang = orc.rope_angles(*grid, *split)
    for h in range(heads):
        sl = slice(h * D, (h + 1) * D)
        L = (orc.apply_rope(q[0, :, sl], ang) @ orc.apply_rope(k[0, :, sl], ang).T) * D ** -0.5
        for qb in range(3):
            for kt in range(5):
                blk = L[qb * 256:(qb + 1) * 256, kt * 128:(kt + 1) * 128]
                assert abs(sc[0, h, qb, kt] - blk.mean()) < 1e-12 * max(1.0, abs(blk).max())


def test_block_selection_matches_a_stable_sort_and_breaks_ties_low():
    scores = rand(3, 17)
    scores[1, [2, 9, 11]] = scores[1].max() + 1.0  # a three-way tie at the top
    sel = orc.anchor_block_select(scores, 5)
    for r in range(3):
        ref = np.sort(np.argsort(-scores[r], kind="stable")[:5])
        assert np.array_equal(sel[r], ref)
    assert {2, 9, 11} <= set(sel[1].tolist())
    assert np.array_equal(orc.anchor_block_select(scores[1:2], 2), [[2, 9]])


def test_tile_restricted_anchor_equals_dense_when_all_kept_and_gathered_softmax():
    grid, split, heads, D = (2, 15, 20), (2, 1, 1), 2, 8
    N = 600
    q, k, v, g = _sparse_inputs(N, heads, D)
    nkt = 5
    all_tiles = np.broadcast_to(np.arange(nkt), (1, heads, 3, nkt))
    dense = orc.softmax_anchor(q, k, v, grid, split, heads, gate=g)
    assert rel(orc.softmax_anchor_tiles(q, k, v, grid, split, heads, all_tiles, gate=g), dense) < 1e-12
    # two tiles per block, different per head and block: each row equals a
    # plain softmax over the gathered keys (naive, no max subtraction)
    tiles = np.array([[[[0, 4], [1, 2], [3, 4]], [[2, 3], [0, 1], [1, 4]]]])
    rows = np.array([0, 255, 256, 511, 599])
    y = orc.softmax_anchor_tiles(q, k, v, grid, split, heads, tiles, rows=rows)
    ang = orc.rope_angles(*grid, *split)
    for h in range(heads):
        sl = slice(h * D, (h + 1) * D)
        qr, kr = orc.apply_rope(q[0, :, sl], ang), orc.apply_rope(k[0, :, sl], ang)
        for ri, i in enumerate(rows):
            keys = np.concatenate([np.arange(t * 128, min((t + 1) * 128, N)) for t in tiles[0, h, i // 256]])
            yn = orc.softmax_naive(qr[i:i + 1], kr[keys], v[0, keys, sl], D ** -0.5)
            assert rel(y[0, ri:ri + 1, sl], yn) < 1e-12


def test_stack_with_every_tile_kept_equals_the_dense_stack():
    grid, split, heads, D = (2, 15, 20), (2, 1, 1), 1, 8
    N, C, layers = 600, 8, 4
    x = rand(1, N, C)
    ws = [{"qkvg": rand(4 * C, C) / np.sqrt(C), "o": rand(C, C) / np.sqrt(C)} for _ in range(layers)]
    dense = orc.hybrid_stack(x, ws, None, None, grid, split, heads, layers, use_attnres=False,
                             ffn=False)
    kept = orc.hybrid_stack(x, ws, None, None, grid, split, heads, layers, use_attnres=False,
                            ffn=False, anchor_keep=5)
    assert rel(kept, dense) < 1e-12


# ------------------------------------------------------------------ AttnRes (P6)

@pytest.mark.parametrize("S,C", [(1, 8), (2, 16), (3, 24), (4, 8)])
def test_attnres_backward_matches_central_finite_differences(S, C):
    B, N = 2, 5
    srcs = [rand(B, N, C) * (1 + i) for i in range(S)]
    w = rand(C)
    dh = rand(B, N, C)
    d_srcs, dw = orc.attnres_route_backward(srcs, w, dh)

    def loss(ss, ww):
        return (orc.attnres_route(ss, ww)[0] * dh).sum()

    h = 1e-6
    for i in range(S):
        u = rand(B, N, C)
        plus = [x + h * u if j == i else x for j, x in enumerate(srcs)]
        minus = [x - h * u if j == i else x for j, x in enumerate(srcs)]
        fd = (loss(plus, w) - loss(minus, w)) / (2 * h)
        assert abs(fd - (d_srcs[i] * u).sum()) <= 1e-7 * max(1.0, abs(fd)), (i, fd)
    u = rand(C)
    fd = (loss(srcs, w + h * u) - loss(srcs, w - h * u)) / (2 * h)
    assert abs(fd - (dw * u).sum()) <= 1e-7 * max(1.0, abs(fd))
    if S == 1:  # one source: h = v, so dv = dh and dw = 0
        assert rel(d_srcs[0], dh) < 1e-14 and np.abs(dw).max() < 1e-12

def test_attnres_two_source_closed_form():
    """C = 4, v1 = a e1 (a > 0), v2 = 0.  RMSNorm(v1) = a e1 / sqrt(a^2/4 + eps),
    RMSNorm(0) = 0.  With w = (L, 0, 0, 0) the logits are
    L * a / sqrt(a^2/4 + eps) and 0, so alpha = softmax of those and
    h = alpha_1 v1."""
    a, L = 3.0, 0.4
    v1 = np.zeros((1, 1, 4)); v1[..., 0] = a
    v2 = np.zeros((1, 1, 4))
    w = np.array([L, 0, 0, 0])
    l1 = L * a / math.sqrt(a * a / 4 + orc.RMS_EPS)
    a1 = math.exp(l1) / (math.exp(l1) + 1.0)
    h, alpha = orc.attnres_route([v1, v2], w)
    np.testing.assert_allclose(alpha[0, 0], [a1, 1 - a1], rtol=1e-14)
    np.testing.assert_allclose(h[0, 0], [a1 * a, 0, 0, 0], rtol=1e-14)


def test_attnres_invariants():
    B, N, C = 2, 7, 32
    srcs = [rand(B, N, C) for _ in range(4)]
    w = rand(C) / math.sqrt(C)
    h, alpha = orc.attnres_route(srcs, w)
    np.testing.assert_allclose(alpha.sum(-1), 1.0, rtol=1e-14)
    # one source: h = v exactly
    h1, a1 = orc.attnres_route(srcs[:1], w)
    assert np.array_equal(h1, srcs[0]) and np.all(a1 == 1.0)
    # permuting the sources permutes alpha and leaves h unchanged
    perm = [2, 0, 3, 1]
    hp, ap = orc.attnres_route([srcs[i] for i in perm], w)
    assert rel(hp, h) < 1e-14
    np.testing.assert_allclose(ap, alpha[..., perm], rtol=1e-13)
    # scaling a source by s > 0 leaves its logit unchanged (up to eps)
    hs, as_ = orc.attnres_route([srcs[0] * 7.0] + srcs[1:], w)
    np.testing.assert_allclose(as_, alpha, rtol=1e-5)
    # w = 0: the mean of the sources
    h0, _ = orc.attnres_route(srcs, np.zeros(C))
    np.testing.assert_allclose(h0, np.mean(srcs, axis=0), rtol=1e-13)


def test_rmsnorm_closed_form():
    x = np.full((1, 8), -2.0)
    np.testing.assert_allclose(orc.rmsnorm(x), -2.0 / math.sqrt(4.0 + orc.RMS_EPS), rtol=1e-15)


# -------------------------------------------------------------------- stack

def test_schedule_matches_page_constants():
    c = json.load(open(os.path.join(GOLDEN, "page_constants.json")))
    lin, soft = c["linear_to_softmax_ratio"]
    ratio = lin + soft
    anchors = [l for l in range(16) if orc.is_anchor_layer(l, ratio)]
    assert anchors == [3, 7, 11, 15]
    assert len(anchors) / 16 == c["softmax_fraction"]
    assert c["attnres_block_span"] == 8 and c["shared_router_queries"] == 2
    v1 = c["v1_model"]
    assert v1["width"] == v1["heads"] * v1["head_dim"] and v1["ffn"] == 3 * v1["width"]


def _zero_stack_weights(layers, C, F):
    return [dict(qkvg=rand(4 * C, C) / math.sqrt(C), o=np.zeros((C, C)),
                 up=rand(F, C) / math.sqrt(C), down=np.zeros((C, F))) for _ in range(layers)]


@pytest.mark.parametrize("layers,span", [(16, 8), (5, 2), (3, 8)])
def test_stack_block_bookkeeping_closed_form(layers, span):
    """With W_o = W_down = 0 every sublayer output is 0, so the partial sum and
    every block summary are 0 (RMSNorm(0) = 0, logit 0).  The output is
    route([x, 0 * nsum]) = x * e^l / (e^l + nsum) with l = w . RMSNorm(x) and
    nsum = layers // span completed summaries (the partial sum is empty after a
    completed block and 0 otherwise, adding one more zero source)."""
    grid, split, heads, D = (2, 2, 2), (1, 1, 2), 2, 8
    C, N = heads * D, 8
    x = rand(1, N, C)
    w_attn, w_ffn = rand(C) / 4, rand(C) / 4
    ws = _zero_stack_weights(layers, C, 3 * C)
    out = orc.hybrid_stack(x, ws, w_attn, w_ffn, grid, split, heads, layers, block_span=span)
    nzero = layers // span + (1 if layers % span else 0)
    lx = orc.rmsnorm(x) @ w_attn
    exp = x * (np.exp(lx) / (np.exp(lx) + nzero))[..., None]
    assert rel(out, exp) < 1e-13


def test_stack_without_attnres_is_residual_composition():
    grid, split, heads, D = (2, 2, 2), (1, 1, 2), 2, 8
    C, N = heads * D, 8
    x = rand(1, N, C)
    ws = [dict(qkvg=rand(4 * C, C) / 4, o=rand(C, C) / 4) for _ in range(4)]
    out = orc.hybrid_stack(x, ws, None, None, grid, split, heads, 4, use_attnres=False, ffn=False)
    ref = x.copy()
    for l in range(4):
        xh = ref / np.sqrt(np.mean(ref ** 2, -1, keepdims=True) + orc.RMS_EPS)
        qkvg = xh @ ws[l]["qkvg"].T
        q, k, v, g = (qkvg[..., i * C:(i + 1) * C] for i in range(4))
        if l == 3:
            a = orc.softmax_anchor(q, k, v, grid, split, heads, gate=g)
        else:
            a = orc.linattn_bruteforce(q, k, v, grid, split, heads, gate=g)
        ref = ref + a @ ws[l]["o"].T
    assert rel(out, ref) < 1e-12


# Textbook values of the logistic function: sigma(1), sigma(2).
SIGMA_1 = 0.7310585786300049
SIGMA_2 = 0.8807970779778823


def test_silu_closed_form_values_and_odd_part():
    """SiLU(x) = x sigma(x): SiLU(0) = 0, SiLU(1) = sigma(1), SiLU(-1) =
    -(1 - sigma(1)), SiLU(2) = 2 sigma(2), SiLU(-2) = -2 (1 - sigma(2)); and
    SiLU(x) - SiLU(-x) = x for every x (sigma(x) + sigma(-x) = 1), which
    x * sigma(-x) or a missing factor of x would break."""
    got = orc.silu(np.array([0.0, 1.0, -1.0, 2.0, -2.0]))
    exp = np.array([0.0, SIGMA_1, -(1 - SIGMA_1), 2 * SIGMA_2, -2 * (1 - SIGMA_2)])
    np.testing.assert_allclose(got, exp, rtol=1e-15, atol=1e-16)
    x = rand(50) * 5
    np.testing.assert_allclose(orc.silu(x) - orc.silu(-x), x, rtol=1e-13, atol=1e-14)
    assert orc.silu(np.array([60.0]))[0] == pytest.approx(60.0, rel=1e-15)
    assert abs(orc.silu(np.array([-60.0]))[0]) < 1e-24


def test_ffn_sublayer_hand_worked():
    """C = 2, hidden 3, asymmetric weights (a transposed W_up or W_down fails):
    x = (1, -2); W_up rows (1, 0), (0, 1), (1, 1) give pre-activations
    (1, -2, -1); u = SiLU of them = (sigma(1), -2 (1 - sigma(2)), -(1 - sigma(1)));
    W_down rows (1, 2, 3), (0, -1, 1) give (u0 + 2 u1 + 3 u2, u2 - u1)."""
    xh = np.array([[1.0, -2.0]])
    Wl = dict(up=np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]]),
              down=np.array([[1.0, 2.0, 3.0], [0.0, -1.0, 1.0]]))
    u0, u1, u2 = SIGMA_1, -2 * (1 - SIGMA_2), -(1 - SIGMA_1)
    exp = np.array([[u0 + 2 * u1 + 3 * u2, u2 - u1]])
    np.testing.assert_allclose(orc._ffn_sublayer(xh, Wl), exp, rtol=1e-14)


def test_stack_ffn_sublayer_enters_the_residual_stream():
    """One layer without AttnRes, W_o = 0, FFN on: x' = x + FFN(RMSNorm x).
    x = (2, -4, 2, -4) has mean square 10, so RMSNorm x = x / sqrt(10 + eps);
    with W_up = I and W_down = 2 I the output is x + 2 SiLU(x / sqrt(10 + eps))."""
    grid, split, heads, D = (1, 1, 1), (0, 0, 1), 2, 2
    C = heads * D
    x = np.array([[[2.0, -4.0, 2.0, -4.0]]])
    ws = [dict(qkvg=rand(4 * C, C), o=np.zeros((C, C)), up=np.eye(C), down=2 * np.eye(C))]
    out = orc.hybrid_stack(x, ws, None, None, grid, split, heads, 1, use_attnres=False, ffn=True)
    r = math.sqrt(10 + orc.RMS_EPS)
    xn = x / r
    exp = x + 2 * xn / (1 + np.exp(-xn))
    np.testing.assert_allclose(out, exp, rtol=1e-14)


# ---------------------------------------------------------------- MX formats (projection GEMMs)

def _decode_e4m3(code):
    """Value of an 8-bit E4M3 code from its fields (None for the NaN codes)."""
    sign, e, m = code >> 7, (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return None
    mag = m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return -mag if sign else mag


def _decode_e2m1(code):
    sign, e, m = code >> 3, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return -mag if sign else mag


def test_mx_element_grids_match_the_bit_layouts_and_torch():
    e4 = sorted({v for c in range(256) if (v := _decode_e4m3(c)) is not None and v >= 0})
    assert np.array_equal(orc.fp_values(orc.E4M3), np.array(e4))
    # torch's float8_e4m3fn, read code by code
    t = torch.arange(128, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(orc.fp_values(orc.E4M3), t[:127]) and np.isnan(t[127])
    e2 = sorted({_decode_e2m1(c) for c in range(16) if _decode_e2m1(c) >= 0})
    assert np.array_equal(orc.fp_values(orc.E2M1), np.array(e2))
    assert orc.fp_values(orc.E2M1).tolist() == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_mx_rounding_matches_torch_float8_including_ties():
    g = np.random.default_rng(7)
    vals = orc.fp_values(orc.E4M3)
    mids = (vals[1:] + vals[:-1]) / 2  # exact ties, representable in float32
    x = np.concatenate([mids, -mids, g.uniform(-448, 448, 4000),
                        g.standard_normal(2000) * 2.0 ** g.integers(-12, 8, 2000)])
    x = np.clip(x, -448, 448).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(orc.round_to_format(x.astype(np.float64), orc.E4M3), ref)


def test_mx_round_e2m1_hand_worked():
    x = [0.2, 0.25, 0.3, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.5, 7.0, -2.5, -0.25]
    # ties go to the even code: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2,
    # 2.5 -> 2, 3.5 -> 4, 5 -> 4; above 6 saturates
    exp = [0.0, 0.0, 0.5, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, -2.0, -0.0]
    assert orc.round_to_format(x, orc.E2M1).tolist() == exp


def test_mx_scale_rule_and_saturation():
    x = np.zeros((1, 32))
    x[0, :4] = [500.0, 1.0, -2.0, 3.0]
    el, s = orc.mx_quantize(x, orc.E4M3)
    # floor(log2 500) = 8 = emax: scale 2^0; 500 saturates to 448
    assert s.tolist() == [[0]] and el[0, :4].tolist() == [448.0, 1.0, -2.0, 3.0]
    el, s = orc.mx_quantize(x, orc.E2M1)
    # floor(log2 500) - 2 = 6: 500 / 64 = 7.8 -> 6, 1/64 -> 0, 3/64 -> 0
    assert s.tolist() == [[6]] and el[0, :4].tolist() == [6.0, 0.0, -0.0, 0.0]
    z, sz = orc.mx_quantize(np.zeros((2, 64)), orc.E4M3)
    assert not z.any() and (sz == orc.MX_SCALE_MIN).all()


def test_mx_quantize_is_invariant_under_power_of_two_scaling():
    x = rand(6, 96)
    for fmt in (orc.E4M3, orc.E2M1):
        el, s = orc.mx_quantize(x, fmt)
        for j in (-20, -3, 5, 31):
            el2, s2 = orc.mx_quantize(x * 2.0 ** j, fmt)
            assert np.array_equal(el2, el) and np.array_equal(s2, s + j)


def test_mx_representable_blocks_round_trip_exactly():
    g = np.random.default_rng(11)
    for fmt in (orc.E4M3, orc.E2M1):
        vals = orc.fp_values(fmt)
        top = vals[vals >= 2.0 ** fmt["emax"]]  # the block max lies in the top binade
        el = g.choice(vals, size=(5, 64)) * g.choice([-1.0, 1.0], size=(5, 64))
        el[:, 0], el[:, 32] = g.choice(top, 5), -g.choice(top, 5)
        s = g.integers(-10, 10, size=(5, 2))
        x = orc.mx_dequantize(el, s)
        el2, s2 = orc.mx_quantize(x, fmt)
        assert np.array_equal(s2, s) and np.array_equal(el2, el)


def test_mx_quantize_error_within_half_an_ulp_or_saturation():
    x = rand(8, 128) * np.exp(rand(8, 128))
    for fmt in (orc.E4M3, orc.E2M1):
        el, s = orc.mx_quantize(x, fmt)
        deq = orc.mx_dequantize(el, s)
        scale = np.repeat(np.exp2(s), 32, axis=-1)
        u = np.abs(x) / scale  # magnitude in element units
        half_ulp = np.exp2(np.floor(np.log2(np.maximum(u, 2.0 ** (1 - fmt["bias"])))) - fmt["mbits"] - 1)
        sat = u > fmt["maxval"]
        err = np.abs(deq - x) / scale
        assert (err[~sat] <= half_ulp[~sat] * (1 + 1e-12)).all()
        assert np.allclose(err[sat], u[sat] - fmt["maxval"], rtol=0, atol=1e-12)
        assert (u < 2.0 ** (fmt["emax"] + 1)).all()  # the scale rule bounds every block


def test_mx_linear_is_the_product_of_the_dequantised_operands():
    g = np.random.default_rng(5)
    M, N, K = 7, 5, 96
    xe = g.choice(orc.fp_values(orc.E4M3), (M, K)) * g.choice([-1, 1], (M, K))
    we = g.choice(orc.fp_values(orc.E2M1), (N, K)) * g.choice([-1, 1], (N, K))
    xe[:, ::32], we[:, ::32] = 448.0, 6.0  # block maxima in the top binade
    x = orc.mx_dequantize(xe, g.integers(-4, 4, (M, K // 32)))
    w = orc.mx_dequantize(we, g.integers(-4, 4, (N, K // 32)))
    # exactly representable operands: the quantised GEMM is the plain product
    assert np.array_equal(orc.mx_linear(x, w), x @ w.T)
    # and on general operands it differs from the plain product by the
    # rounding of each operand only
    a, b = rand(M, K), rand(N, K)
    qa = orc.mx_dequantize(*orc.mx_quantize(a, orc.E4M3))
    qb = orc.mx_dequantize(*orc.mx_quantize(b, orc.E2M1))
    assert np.allclose(orc.mx_linear(a, b), qa @ qb.T, rtol=0, atol=1e-12)
    assert rel(orc.mx_linear(a, b), a @ b.T) < 0.5


def test_error_measures_hand_worked():
    """max_rel_err divides the largest difference by the largest reference
    magnitude; elementwise_rel_err divides each difference by its own
    reference magnitude, floored at 1e-3 of the largest."""
    ref = np.array([10.0, 1.0, -0.001, 0.0])
    got = np.array([10.5, 1.0, -0.002, 0.0])
    assert orc.max_rel_err(got, ref) == pytest.approx(0.05, rel=1e-15)
    # element 2: |0.001| / max(0.001, 0.01) = 0.1; element 0: 0.5 / 10 = 0.05
    assert orc.elementwise_rel_err(got, ref) == pytest.approx(0.1, rel=1e-12)
    got2 = np.array([10.0, 1.0, -0.001, 0.003])   # 0.003 / 0.01
    assert orc.elementwise_rel_err(got2, ref) == pytest.approx(0.3, rel=1e-12)
    assert orc.max_rel_err(got2, ref) == pytest.approx(0.0003, rel=1e-12)


def test_mx_stack_projections_are_the_mx_linear():
    """The stack's MX option changes only the projections: with weights whose
    MX rounding is exact (E2M1 values times a power of two per block), one
    layer without AttnRes and without FFN
    equals the exact layer with the activations' MXFP8 rounding applied to
    the normalised input and to the attention output (quantising along the
    wrong axis, with the wrong format, or skipping a projection fails)."""
    grid, split, heads, D = (2, 2, 2), (2, 3, 3), 2, 16
    C, N = heads * D, 8
    x = rand(1, N, C)
    vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    pick = lambda *sh: rng.choice(vals, size=sh) * rng.choice([-1.0, 1.0], size=sh) * 2.0 ** -3
    ws = [dict(qkvg=pick(4 * C, C), o=pick(C, C))]
    out = orc.hybrid_stack(x, ws, None, None, grid, split, heads, 1, use_attnres=False,
                           ffn=False, mx=True)
    q8 = lambda a: orc.mx_dequantize(*orc.mx_quantize(a, orc.E4M3))
    # the weights are MXFP4-exact: their quantisation is the identity
    wq = orc.mx_dequantize(*orc.mx_quantize(ws[0]["qkvg"], orc.E2M1))
    np.testing.assert_array_equal(wq, ws[0]["qkvg"])
    xh = q8(orc.rmsnorm(x)[0])
    qkvg = xh @ ws[0]["qkvg"].T
    q, k, v, g = (qkvg[None, :, i * C:(i + 1) * C] for i in range(4))
    a = orc.linattn_bruteforce(q, k, v, grid, split, heads, gate=g)
    ref = x + q8(a[0]) @ ws[0]["o"].T
    assert rel(out, ref) < 1e-12
