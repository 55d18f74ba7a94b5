"""Float64 CPU oracle for the hybrid linear-softmax attention hot path.

TEST INFRASTRUCTURE ONLY.  This module is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py``; nothing in the product package imports or executes it,
and it imports nothing from the product package.  It is plain numpy in
float64: every function follows one passage of the pages, in the pages' order
and notation, with no blocking, fusion or reordering beyond what that passage
states.  A matrix product (``@`` / ``einsum``) is used as a library step.

Sources (cited by page title and section / equation):

* [SV1] "SANA-Video: Efficient Video Generation with Block Linear Diffusion
  Transformer" (paper notes), sec. 3.2 "Linear Attention with RoPE" (the
  equation for O_i, and the linear-attention-with-RoPE pseudocode), sec. 3.4
  "Block Linear Attention with Constant-Memory KV Cache" (the causal equation
  for O_i, the cumulative-sum state, the complexity table and Algorithm 1),
  sec. 4.1 (model configuration table).
* [SV2] "SANA-Video 2.0" (hyper.ai summary of arXiv 2607.21553), Method,
  "Hybrid attention and block residuals" paragraph and its AttnRes equation
  h_l = sum_i alpha_{i->l} v_i, alpha = softmax_i((w + phi_tau(t))^T RMSNorm(v_i));
  the shared-router-query paragraph; Experiments (timestep-free router,
  block span 8).
* [SV2-abs] "SANA-Video 2.0" abstract (ai-pulse-lab page): gated linear
  attention with gated softmax anchors at a 3:1 ratio.

Readings where the pages are silent:

* 3D RoPE layout: global pair j rotates elements (2j, 2j+1); pairs
  [0, n_t) use the frame index t, the next n_h the row index h, the last n_w
  the column index w; within an axis, local pair k has angle
  pos * theta**(-k / n_axis), theta = 10000; rotation (x, y) ->
  (x cos - y sin, x sin + y cos).  Positions are integer grid indices from 0,
  the frame index being absolute (t_offset + local frame).
* eps = 1e-6 added to the denominator after the dot product ([SV1] sec. 3.2
  pseudocode names eps without a value).
* "Gated" = elementwise sigmoid of gate logits G = x W_g on the output.
* Block-causal: a block sees the whole of itself plus every earlier block
  (Algorithm 1 updates the cache only after the block is fully denoised);
  RoPE sits in the numerator exactly as in the bidirectional form.
* Softmax anchor: the same 3D RoPE applied to raw Q and K (no ReLU),
  scale 1/sqrt(D), bidirectional.
* AttnRes: RMSNorm without gain, eps_r = 1e-6, phi_tau(t) = 0; sources in the
  order [embedding, block summaries..., running partial sum], the partial sum
  left out while it is empty.
* Stack: layer l is an anchor iff l % 4 == 3; FFN = W_down SiLU(W_up x) with
  hidden size ffn_mult * C; sublayer input RMSNorm(h) without gain.
* Backward: the pages train from scratch ([SV1] sec. 4 training setup) but
  print no backward; linattn_backward is the chain rule through the forward
  as written (ReLU derivative 1 for x > 0, 0 otherwise), pinned by finite
  differences.
* MX formats ([SV2] Experiments name MXFP4 weights and MXFP8 activations
  for the linear GEMMs): the OCP Microscaling v1.0 definitions.
  - Blocks are 32 elements along the contraction axis, with one E8M0
    exponent s = floor(log2 amax) - emax_elem.
  - Elements are E4M3 (max 448) or E2M1 (max 6), rounded to nearest-even
    and saturated.
* Sparse anchor ([SV2] Experiments and [SV2-abs] say only that the
  deployment stack applies sparse attention to the softmax anchors): queries
  in blocks of 256 tokens, keys in tiles of 128; each block keeps the `keep`
  key tiles with the largest pooled logit mean(RoPE(Q) * scale) .
  mean(RoPE(K)) (ties to the lower tile index) and attends to exactly those
  keys.

Parity status: every function here is pinned by tests/test_oracle_pins.py
against brute force, closed forms or invariants, except the absolute values
that only the readings above fix (RoPE layout and frequencies, eps values,
the anchor's use of RoPE, the FFN form, the empty-partial-sum and last-chunk
rules, and the whole block-sparse pattern of the sparse anchor): those are
"parity unpinned" beyond the readings themselves.
"""

from __future__ import annotations

import numpy as np

THETA = 10000.0
EPS = 1e-6
RMS_EPS = 1e-6


# --------------------------------------------------------------------------
# feature map and 3D RoPE  ([SV1] sec. 3.2)
# --------------------------------------------------------------------------

def phi(x):
    """Kernel feature map phi(x) = ReLU(x) ([SV1] sec. 3.2)."""
    return np.maximum(x, 0.0)


def token_grid(T, H, W, t_offset=0):
    """Integer (t, h, w) of every token, token n = (t*H + h)*W + w.

    The frame index is absolute: t_offset + local frame."""
    n = np.arange(T * H * W)
    t = n // (H * W) + t_offset
    h = (n // W) % H
    w = n % W
    return t, h, w


def rope_angles(T, H, W, n_t, n_h, n_w, t_offset=0, theta=THETA):
    """Angle of every (token, rotary pair): array [N, n_t + n_h + n_w].

    Pair j < n_t follows axis t with local index k = j; the next n_h pairs
    follow h, the last n_w follow w; angle = pos * theta**(-k / n_axis)."""
    t, h, w = token_grid(T, H, W, t_offset)
    cols = []
    for pos, n_ax in ((t, n_t), (h, n_h), (w, n_w)):
        k = np.arange(n_ax, dtype=np.float64)
        freq = theta ** (-k / n_ax) if n_ax > 0 else k
        cols.append(pos.astype(np.float64)[:, None] * freq[None, :])
    return np.concatenate(cols, axis=1)


def apply_rope(x, angles):
    """Rotate pairs (2j, 2j+1) of the last axis of x[..., N, D] by angles[N, D/2]."""
    xe = x[..., 0::2]
    xo = x[..., 1::2]
    c = np.cos(angles)
    s = np.sin(angles)
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _heads(x, heads):
    """(B, N, C) -> (B, heads, N, D)."""
    B, N, C = x.shape
    return x.reshape(B, N, heads, C // heads).transpose(0, 2, 1, 3)


def _merge(x):
    """(B, heads, N, D) -> (B, N, C)."""
    B, h, N, D = x.shape
    return x.transpose(0, 2, 1, 3).reshape(B, N, h * D)


# --------------------------------------------------------------------------
# bidirectional ReLU linear attention with RoPE after the ReLU
# ([SV1] sec. 3.2, equation for O_i and the pseudocode)
# --------------------------------------------------------------------------

def linattn_state(k, v, angles, heads):
    """S = sum_j RoPE(phi(K_j))^T V_j  [B, heads, D, D];  z = sum_j phi(K_j)  [B, heads, D].

    The state of [SV1] sec. 3.4 (cumulative sum of S_j and of phi(K_j)^T)."""
    kh = _heads(np.asarray(k, np.float64), heads)
    vh = _heads(np.asarray(v, np.float64), heads)
    k_phi = phi(kh)
    k_rope = apply_rope(k_phi, angles)
    S = np.swapaxes(k_rope, -1, -2) @ vh          # sum_j RoPE(phi K_j)^T V_j
    z = k_phi.sum(axis=2)
    return S, z


def linattn_apply(q, S, z, angles, heads, gate=None, eps=EPS):
    """O_i = RoPE(phi(Q_i)) S / (phi(Q_i) . z + eps);  Y = sigmoid(G) * O.

    Numerator with RoPE, denominator without it ([SV1] sec. 3.2)."""
    qh = _heads(np.asarray(q, np.float64), heads)
    q_phi = phi(qh)
    q_rope = apply_rope(q_phi, angles)
    num = q_rope @ S                               # RoPE(phi Q_i) S
    den = (q_phi @ z[..., :, None])[..., 0]        # phi Q_i . z
    out = _merge(num / (den[..., None] + eps))
    if gate is not None:
        out = sigmoid(np.asarray(gate, np.float64)) * out
    return out


def linattn_bidirectional(q, k, v, grid, rope_split, heads, gate=None, eps=EPS,
                          t_offset=0):
    """One gated bidirectional linear-attention layer on (B, N, C) inputs.

    grid = (T, H, W); rope_split = (n_t, n_h, n_w).  Returns (Y, S, z)."""
    T, H, W = grid
    ang = rope_angles(T, H, W, *rope_split, t_offset=t_offset)
    S, z = linattn_state(k, v, ang, heads)
    y = linattn_apply(q, S, z, ang, heads, gate, eps)
    return y, S, z


def rope_transpose(x, angles):
    """Inverse (= transpose) of apply_rope: rotate pairs by -angle."""
    return apply_rope(x, -angles)


def linattn_backward(q, k, v, grid, rope_split, heads, dy, gate=None, eps=EPS, t_offset=0):
    """Gradients of linattn_bidirectional's Y with respect to Q, K, V and G.

    The forward ([SV1] sec. 3.2, gated per [SV2-abs]) differentiated step by
    step in reverse; the pages train the model from scratch but print no
    backward, so this is the chain rule applied to the forward as written:
      o_i = num_i / den_i, num_i = q'_i S, den_i = phi(q_i) . z + eps,
      y_i = sigmoid(g_i) * o_i.
    Returns (dQ, dK, dV, dG) with dG None when there is no gate."""
    T, H, W = grid
    ang = rope_angles(T, H, W, *rope_split, t_offset=t_offset)
    qh = _heads(np.asarray(q, np.float64), heads)
    kh = _heads(np.asarray(k, np.float64), heads)
    vh = _heads(np.asarray(v, np.float64), heads)
    dyh = _heads(np.asarray(dy, np.float64), heads)
    q_phi, k_phi = phi(qh), phi(kh)
    q_rope, k_rope = apply_rope(q_phi, ang), apply_rope(k_phi, ang)
    S = np.swapaxes(k_rope, -1, -2) @ vh
    z = k_phi.sum(axis=2)
    num = q_rope @ S
    den = (q_phi @ z[..., :, None])[..., 0] + eps
    o = num / den[..., None]
    if gate is not None:
        sg = sigmoid(_heads(np.asarray(gate, np.float64), heads))
        dg = dyh * o * sg * (1.0 - sg)
        do = dyh * sg
    else:
        dg = None
        do = dyh
    dnum = do / den[..., None]                        # d/d num_i
    dden = -(do * o).sum(axis=-1) / den               # d/d den_i
    dq_rope = dnum @ np.swapaxes(S, -1, -2)           # d/d q'_i = dnum_i S^T
    dS = np.swapaxes(q_rope, -1, -2) @ dnum           # sum_i q'_i^T dnum_i
    dz = (dden[..., None] * q_phi).sum(axis=2)        # sum_i dden_i phi(q_i)
    dq_phi = rope_transpose(dq_rope, ang) + dden[..., None] * z[..., None, :]
    dk_rope = vh @ np.swapaxes(dS, -1, -2)            # d/d k'_j = v_j dS^T
    dv = k_rope @ dS                                  # d/d v_j = k'_j dS
    dk_phi = rope_transpose(dk_rope, ang) + dz[..., None, :]
    dq = dq_phi * (qh > 0)
    dk = dk_phi * (kh > 0)
    return _merge(dq), _merge(dk), _merge(dv), None if dg is None else _merge(dg)


def linattn_bruteforce(q, k, v, grid, rope_split, heads, gate=None, eps=EPS,
                       mask=None, t_offset=0):
    """O(N^2) pairwise form of the same layer (pin P1 / P2).

    O_i = sum_j (RoPE(phi Q_i) . RoPE(phi K_j)) V_j / (sum_j phi Q_i . phi K_j + eps),
    with an optional boolean mask[i, j] selecting the visible keys."""
    T, H, W = grid
    ang = rope_angles(T, H, W, *rope_split, t_offset=t_offset)
    qh = _heads(np.asarray(q, np.float64), heads)
    kh = _heads(np.asarray(k, np.float64), heads)
    vh = _heads(np.asarray(v, np.float64), heads)
    q_phi, k_phi = phi(qh), phi(kh)
    q_rope, k_rope = apply_rope(q_phi, ang), apply_rope(k_phi, ang)
    A_num = np.einsum('bhid,bhjd->bhij', q_rope, k_rope)
    A_den = np.einsum('bhid,bhjd->bhij', q_phi, k_phi)
    if mask is not None:
        A_num = A_num * mask
        A_den = A_den * mask
    num = np.einsum('bhij,bhje->bhie', A_num, vh)
    den = A_den.sum(axis=-1)
    out = _merge(num / (den[..., None] + eps))
    if gate is not None:
        out = sigmoid(np.asarray(gate, np.float64)) * out
    return out


# --------------------------------------------------------------------------
# block-causal form with a constant-memory state ([SV1] sec. 3.4, Algorithm 1)
# --------------------------------------------------------------------------

def linattn_block_causal_step(q, k, v, chunk_grid, t_offset, rope_split, heads,
                              S_prev, z_prev, gate=None, eps=EPS, commit=True):
    """One block of the block-causal recurrence.

    The block's own (S_c, z_c) are added to the cumulative state; its output
    uses (S_prev + S_c, z_prev + z_c), i.e. the block sees every earlier block
    and the whole of itself.  With commit the cumulative state is returned as
    the new state (the cache update after the last denoising step of
    Algorithm 1); without it the previous state is returned unchanged.
    Returns (Y, S_new, z_new)."""
    T, H, W = chunk_grid
    ang = rope_angles(T, H, W, *rope_split, t_offset=t_offset)
    S_c, z_c = linattn_state(k, v, ang, heads)
    S_tot = np.asarray(S_prev, np.float64) + S_c
    z_tot = np.asarray(z_prev, np.float64) + z_c
    y = linattn_apply(q, S_tot, z_tot, ang, heads, gate, eps)
    if commit:
        return y, S_tot, z_tot
    return y, np.array(S_prev, np.float64), np.array(z_prev, np.float64)


def linattn_block_causal_sequence(q, k, v, grid, chunk_frames, t_offset, rope_split, heads,
                                  S_prev, z_prev, gate=None, eps=EPS, commit=True):
    """A whole sequence of blocks ([SV1] sec. 3.4, Algorithm 1), each of
    `chunk_frames` frames except a shorter last block when the frame count is
    not a multiple of it (reading: the remainder forms the final block).

    The blocks go through linattn_block_causal_step in order, each committing
    its contribution so that the next block sees it; with commit the state
    after the last block is returned, otherwise the initial state.
    Returns (Y, S, z)."""
    T, H, W = grid
    hw = H * W
    S = np.asarray(S_prev, np.float64)
    z = np.asarray(z_prev, np.float64)
    ys = []
    t0 = 0
    while t0 < T:
        f = min(chunk_frames, T - t0)
        sl = slice(t0 * hw, (t0 + f) * hw)
        y, S, z = linattn_block_causal_step(
            q[:, sl], k[:, sl], v[:, sl], (f, H, W), t_offset + t0, rope_split, heads, S, z,
            gate=None if gate is None else gate[:, sl], eps=eps, commit=True)
        ys.append(y)
        t0 += f
    B, _, C = np.asarray(v).shape
    y = np.concatenate(ys, axis=1) if ys else np.zeros((B, 0, C))
    if commit:
        return y, S, z
    return y, np.array(S_prev, np.float64), np.array(z_prev, np.float64)


def linattn_token_recurrence(q, k, v, grid, rope_split, heads, eps=EPS):
    """Per-token causal recurrence of [SV1] sec. 3.4 (chunk size 1), with RoPE
    in the numerator: O_i = RoPE(phi Q_i)(sum_{j<i} S_j + S_i) / (phi Q_i (sum_{j<=i} phi K_j) + eps)."""
    T, H, W = grid
    ang = rope_angles(T, H, W, *rope_split)
    qh = _heads(np.asarray(q, np.float64), heads)
    kh = _heads(np.asarray(k, np.float64), heads)
    vh = _heads(np.asarray(v, np.float64), heads)
    B, nh, N, D = qh.shape
    out = np.zeros_like(vh)
    S = np.zeros((B, nh, D, vh.shape[-1]))
    z = np.zeros((B, nh, D))
    q_phi, k_phi = phi(qh), phi(kh)
    q_rope, k_rope = apply_rope(q_phi, ang), apply_rope(k_phi, ang)
    for i in range(N):
        S = S + np.einsum('bhd,bhe->bhde', k_rope[:, :, i], vh[:, :, i])
        z = z + k_phi[:, :, i]
        num = np.einsum('bhd,bhde->bhe', q_rope[:, :, i], S)
        den = np.einsum('bhd,bhd->bh', q_phi[:, :, i], z)
        out[:, :, i] = num / (den[..., None] + eps)
    return _merge(out)


# --------------------------------------------------------------------------
# gated softmax anchor ([SV2-abs]; reading: same 3D RoPE on raw Q, K)
# --------------------------------------------------------------------------

def softmax_anchor(q, k, v, grid, rope_split, heads, gate=None, scale=None,
                   rows=None, use_rope=True, t_offset=0):
    """Y = sigmoid(G) * softmax(RoPE(Q) RoPE(K)^T * scale) V over all keys.

    rows: optional index array of query tokens to evaluate (the others are
    not computed); the result then has shape (B, len(rows), C).
    Max-subtracted softmax.  With use_rope=False grid and rope_split are unused."""
    qh = _heads(np.asarray(q, np.float64), heads)
    kh = _heads(np.asarray(k, np.float64), heads)
    vh = _heads(np.asarray(v, np.float64), heads)
    D = qh.shape[-1]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    if use_rope:
        ang = rope_angles(*grid, *rope_split, t_offset=t_offset)
        qh = apply_rope(qh, ang)
        kh = apply_rope(kh, ang)
    if rows is not None:
        qh = qh[:, :, rows]
    logits = (qh @ np.swapaxes(kh, -1, -2)) * scale
    m = logits.max(axis=-1, keepdims=True)
    p = np.exp(logits - m)
    p = p / p.sum(axis=-1, keepdims=True)
    out = _merge(p @ vh)
    if gate is not None:
        g = np.asarray(gate, np.float64)
        if rows is not None:
            g = g[:, rows]
        out = sigmoid(g) * out
    return out


# --------------------------------------------------------------------------
# block-sparse softmax anchor (reading of [SV2] Experiments / [SV2-abs]:
# the deployment stack applies sparse attention to the softmax anchors; the
# pages give no pattern)
# --------------------------------------------------------------------------

Q_BLOCK = 256   # query rows per block (reading)
K_TILE = 128    # keys per tile (reading)


def anchor_block_scores(q, k, grid, rope_split, heads, scale=None, t_offset=0):
    """Pooled-logit score of every (query block, key tile) pair.

    Reading: q_bar = mean over the block's tokens of RoPE(Q) * scale, k_bar =
    mean over the tile's tokens of RoPE(K); score = q_bar . k_bar (the mean
    logit of the block pair).  Returns [B, heads, n_qblocks, n_ktiles]."""
    qh = _heads(np.asarray(q, np.float64), heads)
    kh = _heads(np.asarray(k, np.float64), heads)
    D = qh.shape[-1]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    ang = rope_angles(*grid, *rope_split, t_offset=t_offset)
    qh = apply_rope(qh, ang) * scale
    kh = apply_rope(kh, ang)
    N = qh.shape[2]
    nqb = -(-N // Q_BLOCK)
    nkt = -(-N // K_TILE)
    qbar = np.stack([qh[:, :, i * Q_BLOCK:(i + 1) * Q_BLOCK].mean(axis=2) for i in range(nqb)], axis=2)
    kbar = np.stack([kh[:, :, t * K_TILE:(t + 1) * K_TILE].mean(axis=2) for t in range(nkt)], axis=2)
    return qbar @ np.swapaxes(kbar, -1, -2)


def anchor_block_select(scores, keep):
    """Top-`keep` key tiles of every query block by score, ties to the lower
    tile index, returned in ascending tile order: int array [..., keep]."""
    scores = np.asarray(scores, np.float64)
    lead = scores.shape[:-1]
    n = scores.shape[-1]
    flat = scores.reshape(-1, n)
    out = np.empty((flat.shape[0], keep), np.int64)
    for r in range(flat.shape[0]):
        order = sorted(range(n), key=lambda t: (-flat[r, t], t))
        out[r] = sorted(order[:keep])
    return out.reshape(*lead, keep)


def softmax_anchor_tiles(q, k, v, grid, rope_split, heads, tiles, gate=None, scale=None,
                         rows=None, t_offset=0):
    """The gated softmax anchor with each query restricted to the keys of the
    tiles kept for its block: tiles [B, heads, n_qblocks, keep] (distinct
    indices of 128-key tiles).  Softmax over exactly those keys."""
    qh = _heads(np.asarray(q, np.float64), heads)
    kh = _heads(np.asarray(k, np.float64), heads)
    vh = _heads(np.asarray(v, np.float64), heads)
    B, nh, N, D = qh.shape
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    ang = rope_angles(*grid, *rope_split, t_offset=t_offset)
    qh = apply_rope(qh, ang)
    kh = apply_rope(kh, ang)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.zeros((B, nh, len(rows), D))
    key_tile = np.arange(N) // K_TILE
    for b in range(B):
        for h in range(nh):
            for ri, i in enumerate(rows):
                allowed = np.isin(key_tile, tiles[b, h, i // Q_BLOCK])
                lg = (kh[b, h, allowed] @ qh[b, h, i]) * scale
                p = np.exp(lg - lg.max())
                out[b, h, ri] = (p / p.sum()) @ vh[b, h, allowed]
    out = _merge(out)
    if gate is not None:
        out = sigmoid(np.asarray(gate, np.float64)[:, rows]) * out
    return out


def softmax_naive(q, k, v, scale):
    """Naive softmax attention without max subtraction, single head (pin P5)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    e = np.exp((q @ k.T) * scale)
    return (e / e.sum(axis=1, keepdims=True)) @ v


# --------------------------------------------------------------------------
# Block Attention Residuals router ([SV2] AttnRes equation)
# --------------------------------------------------------------------------

def rmsnorm(x, eps=RMS_EPS):
    """RMSNorm without gain over the last axis."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def attnres_route(sources, w, eps=RMS_EPS):
    """h = sum_i alpha_i v_i with alpha = softmax_i(w^T RMSNorm(v_i)).

    sources: list of (B, N, C) arrays in the order [embedding, block
    summaries..., partial sum]; w: (C,) router query (phi_tau(t) = 0).
    Returns (h, alpha) with alpha of shape (B, N, len(sources))."""
    V = np.stack([np.asarray(s, np.float64) for s in sources], axis=-2)  # B,N,S,C
    w = np.asarray(w, np.float64)
    logits = rmsnorm(V, eps) @ w                                       # B,N,S
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    alpha = e / e.sum(axis=-1, keepdims=True)
    h = np.einsum('bns,bnsc->bnc', alpha, V)
    return h, alpha


def attnres_route_backward(sources, w, dh, eps=RMS_EPS):
    """Gradients of attnres_route's h with respect to the sources and w, given
    dh: the chain rule through the forward as written (the pages print no
    backward).  With r_i = sqrt(mean_c v_i^2 + eps) and l_i = w . v_i / r_i:
      d alpha_i = dh . v_i,  d l_i = alpha_i (d alpha_i - sum_j alpha_j d alpha_j),
      d v_i = alpha_i dh + d l_i (w / r_i - l_i v_i / (C r_i^2)),
      d w = sum over tokens of sum_i d l_i v_i / r_i.
    Returns (list of d v_i, d w)."""
    V = np.stack([np.asarray(s, np.float64) for s in sources], axis=-2)  # B,N,S,C
    w = np.asarray(w, np.float64)
    dh = np.asarray(dh, np.float64)
    C = V.shape[-1]
    r = np.sqrt(np.mean(V * V, axis=-1) + eps)                          # B,N,S
    logits = (V @ w) / r
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    alpha = e / e.sum(axis=-1, keepdims=True)
    dalpha = np.einsum('bnc,bnsc->bns', dh, V)
    dl = alpha * (dalpha - (alpha * dalpha).sum(axis=-1, keepdims=True))
    dV = (alpha[..., None] * dh[..., None, :]
          + dl[..., None] * (w / r[..., None] - (logits / (C * r * r))[..., None] * V))
    dw = np.einsum('bns,bnsc->c', dl / r, V)
    return [dV[..., i, :] for i in range(V.shape[-2])], dw


# --------------------------------------------------------------------------
# hybrid stack ([SV2] method paragraph; [SV2-abs] 3:1 interleave)
# --------------------------------------------------------------------------

def silu(x):
    return x * sigmoid(x)


def is_anchor_layer(l, ratio=4):
    """Layer l (0-based) is a softmax anchor iff l % ratio == ratio - 1."""
    return l % ratio == ratio - 1


def _project(x, W, mx=False):
    """x W^T: exact, or the MX projection Q8(x) Q4(W)^T ([SV2] Experiments:
    the deployment quantises the linear GEMMs, MXFP8 activations and MXFP4
    weights) through mx_linear, blocked along the contraction axis."""
    W = np.asarray(W, np.float64)
    if not mx:
        return x @ W.T
    lead = x.shape[:-1]
    return mx_linear(np.asarray(x, np.float64).reshape(-1, x.shape[-1]), W).reshape(*lead, -1)


def _attention_sublayer(xh, Wl, grid, rope_split, heads, eps, anchor, anchor_keep=0, mx=False):
    C = xh.shape[-1]
    qkvg = _project(xh, Wl['qkvg'], mx)
    q, k, v, g = (qkvg[..., i * C:(i + 1) * C] for i in range(4))
    if anchor and anchor_keep > 0:
        tiles = anchor_block_select(anchor_block_scores(q, k, grid, rope_split, heads), anchor_keep)
        a = softmax_anchor_tiles(q, k, v, grid, rope_split, heads, tiles, gate=g)
    elif anchor:
        a = softmax_anchor(q, k, v, grid, rope_split, heads, gate=g)
    else:
        a, _, _ = linattn_bidirectional(q, k, v, grid, rope_split, heads, gate=g, eps=eps)
    return _project(a, Wl['o'], mx)


def _ffn_sublayer(xh, Wl, mx=False):
    u = silu(_project(xh, Wl['up'], mx))
    return _project(u, Wl['down'], mx)


def hybrid_stack(x, weights, w_attn, w_ffn, grid, rope_split, heads, layers,
                 block_span=8, ratio=4, use_attnres=True, ffn=True, eps=EPS,
                 rms_eps=RMS_EPS, anchor_keep=0, mx=False):
    """Forward of the hybrid stack.

    With AttnRes: every sublayer reads h = route(V_l) over [embedding,
    completed block summaries, running partial sum], its output is added to
    the partial sum, and after every block_span layers the partial sum is
    frozen as a block summary.  The result is the representation a next layer
    would read: route(V, w_attn) over the final source set.
    Without AttnRes: plain pre-norm residual x += sublayer(RMSNorm(x)).
    anchor_keep > 0: the anchors are block-sparse (anchor_block_select's tiles).
    mx: every projection (QKVG, O, FFN up and down) is the MX projection
    (mx_linear); attention, routes and norms stay exact."""
    x = np.asarray(x, np.float64)
    if not use_attnres:
        for l in range(layers):
            Wl = weights[l]
            x = x + _attention_sublayer(rmsnorm(x, rms_eps), Wl, grid, rope_split,
                                        heads, eps, is_anchor_layer(l, ratio), anchor_keep, mx)
            if ffn:
                x = x + _ffn_sublayer(rmsnorm(x, rms_eps), Wl, mx)
        return x
    summaries = []
    partial = None

    def sources():
        return [x] + summaries + ([partial] if partial is not None else [])

    for l in range(layers):
        Wl = weights[l]
        h, _ = attnres_route(sources(), w_attn, rms_eps)
        out = _attention_sublayer(rmsnorm(h, rms_eps), Wl, grid, rope_split, heads,
                                  eps, is_anchor_layer(l, ratio), anchor_keep, mx)
        partial = out if partial is None else partial + out
        if ffn:
            h, _ = attnres_route(sources(), w_ffn, rms_eps)
            partial = partial + _ffn_sublayer(rmsnorm(h, rms_eps), Wl, mx)
        if (l + 1) % block_span == 0:
            summaries.append(partial)
            partial = None
    h, _ = attnres_route(sources(), w_attn, rms_eps)
    return h


# --------------------------------------------------------------------------
# MX block-scaled formats for the projection GEMMs  ([SV2] Experiments:
# low-precision inference quantises only the linear GEMM layers, weights to
# MXFP4 and activations to MXFP8; attention stays bf16)
# --------------------------------------------------------------------------

# The pages name the formats without defining them.  Reading: the OCP
# Microscaling (MX) v1.0 definitions.  A block of 32 consecutive elements
# along the contraction axis shares one scale 2^s (an E8M0 exponent,
# s in [-127, 127]).  Each element is an FP8 E4M3 value (MXFP8) or an FP4 E2M1
# value (MXFP4).
E4M3 = {"name": "e4m3", "mbits": 3, "bias": 7, "emax": 8, "maxval": 448.0}
E2M1 = {"name": "e2m1", "mbits": 1, "bias": 1, "emax": 2, "maxval": 6.0}
MX_BLOCK = 32
MX_SCALE_MIN, MX_SCALE_MAX = -127, 127


def fp_values(fmt):
    """The non-negative finite values of an element format, in code order.

    Subnormals are m * 2^(1 - bias - mbits), for m < 2^mbits. Normals are
    (1 + m / 2^mbits) * 2^(e - bias), for biased exponents e >= 1. The list
    stops at the format's largest finite value."""
    mb, bias = fmt["mbits"], fmt["bias"]
    vals = [m * 2.0 ** (1 - bias - mb) for m in range(2 ** mb)]
    e = 1
    while True:
        for m in range(2 ** mb):
            v = (1 + m / 2 ** mb) * 2.0 ** (e - bias)
            if v > fmt["maxval"]:
                return np.array(vals)
            vals.append(v)
        e += 1


def round_to_format(x, fmt):
    """Round to the nearest value of the element format.

    Ties go to the even code, and a magnitude above the largest finite value
    saturates to it. Consecutive non-negative values have consecutive codes,
    so an even index in fp_values is an even code."""
    x = np.asarray(x, np.float64)
    vals = fp_values(fmt)
    a = np.minimum(np.abs(x), fmt["maxval"])
    i = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)  # vals[i-1] < a <= vals[i]
    lo, hi = vals[i - 1], vals[i]
    up = (a - lo > hi - a) | ((a - lo == hi - a) & (i % 2 == 0))
    return np.sign(x) * np.where(up, hi, lo)


def mx_quantize(x, fmt, block=MX_BLOCK):
    """MX quantisation along the last axis, which is the contraction axis.

    Each block of `block` elements gets the exponent
    s = floor(log2(max |x|)) - emax(fmt), clamped to the E8M0 range. An
    all-zero block takes the smallest exponent. The elements are x / 2^s,
    rounded by round_to_format. Returns (elements, s), with s of shape
    x.shape[:-1] + (K / block,)."""
    x = np.asarray(x, np.float64)
    K = x.shape[-1]
    assert K % block == 0, "the contraction length must be a multiple of the block"
    xb = x.reshape(*x.shape[:-1], K // block, block)
    amax = np.max(np.abs(xb), axis=-1)
    _, ex = np.frexp(amax)  # amax = f * 2^ex with f in [1/2, 1): floor(log2 amax) = ex - 1
    s = np.where(amax > 0, ex - 1 - fmt["emax"], MX_SCALE_MIN)
    s = np.clip(s, MX_SCALE_MIN, MX_SCALE_MAX).astype(np.int64)
    el = round_to_format(xb / np.exp2(s)[..., None], fmt)
    return el.reshape(x.shape), s


def mx_dequantize(el, s, block=MX_BLOCK):
    """Elements times their block's scale."""
    el = np.asarray(el, np.float64)
    K = el.shape[-1]
    eb = el.reshape(*el.shape[:-1], K // block, block)
    return (eb * np.exp2(s)[..., None]).reshape(el.shape)


def mx_linear(x, w, block=MX_BLOCK):
    """The quantised projection y = Q8(x) Q4(w)^T.

    Activations x (M, K) are MXFP8 (E4M3 elements). Weights w (N, K) are
    MXFP4 (E2M1 elements). Both are blocked along K, and the dequantised
    operands are multiplied in float64."""
    xq = mx_dequantize(*mx_quantize(x, E4M3, block), block)
    wq = mx_dequantize(*mx_quantize(w, E2M1, block), block)
    return xq @ wq.T


# --------------------------------------------------------------------------
# error measure
# --------------------------------------------------------------------------

def max_rel_err(got, ref):
    """max_i |got_i - ref_i| / max_i |ref_i| (the parity measure)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    denom = np.max(np.abs(ref))
    if denom == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref)) / denom)


def elementwise_rel_err(got, ref, floor=1e-3):
    """max_i |got_i - ref_i| / max(|ref_i|, floor * max_j |ref_j|): the
    elementwise companion of max_rel_err, which also sees errors in outputs
    far smaller than the tensor's largest (e.g. elements gated towards 0)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    a = np.abs(ref)
    m = np.max(a) if a.size else 0.0
    if m == 0.0:
        return float(np.max(np.abs(got))) if got.size else 0.0
    return float(np.max(np.abs(got - ref) / np.maximum(a, floor * m)))
