"""GPU parity of the linear-attention backward (sana_linattn_bwd) against the
float64 oracle's chain-rule gradients (itself pinned by finite differences).

Bar: max relative error <= 2e-2 per gradient tensor (bf16 inputs, bf16
operands of the tensor-core products, fp32 accumulation)."""

import numpy as np
import pytest
import torch

import sana_inputs as si
from oracle import sana_oracle as orc
from tests._sana import sana

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


def f64(t):
    return si.as_f64(t)


def run(B, grid, heads, split, seed, gated=True):
    T, H, W = grid
    N = T * H * W
    C = heads * 128
    q, k, v, g, dy = (si.normal(seed + i, (B, N, C)) for i in range(5))
    if not gated:
        g = None
    rope = sana.Rope(T, H, W, split)
    grads = sana.linattn_bwd(q.cuda(), k.cuda(), v.cuda(), None if g is None else g.cuda(), rope,
                             grid, heads, dy.cuda())
    sana.sync_status()
    ref = orc.linattn_backward(f64(q), f64(k), f64(v), grid, split, heads, f64(dy),
                               gate=None if g is None else f64(g))
    return [None if x is None else x.cpu() for x in grads], ref


@pytest.mark.parametrize("B,grid,heads,split,gated", [
    (2, (3, 9, 16), 2, (22, 21, 21), True),    # N = 432: 3 full tiles + 48 rows
    (1, (6, 7, 19), 1, (20, 22, 22), True),    # N = 798, general rotary split
    (2, (3, 9, 16), 2, (22, 21, 21), False),   # ungated
])
def test_small_ragged_matches_the_oracle(B, grid, heads, split, gated):
    grads, ref = run(B, grid, heads, split, 9700, gated)
    for name, gg, rr in zip(("dq", "dk", "dv", "dg"), grads, ref):
        if rr is None:
            assert gg is None
            continue
        e = orc.max_rel_err(f64(gg), rr)
        assert e <= BF16_TOL, (name, e)


def test_saved_state_equals_recomputed_state():
    """The backward given the forward's (S, z) (sana_linattn_bwd_saved_state)
    runs the same kernels on the same state as the one that rebuilds it."""
    grid, heads = (3, 9, 16), 2
    N = grid[0] * grid[1] * grid[2]
    q, k, v, g, dy = (si.normal(9720 + i, (1, N, heads * 128)).cuda() for i in range(5))
    rope = sana.Rope(*grid, (22, 21, 21))
    S, z = sana.linattn_state(k, v, rope, grid, heads)
    a = sana.linattn_bwd(q, k, v, g, rope, grid, heads, dy)
    b = sana.linattn_bwd(q, k, v, g, rope, grid, heads, dy, S=S, z=z)
    sana.sync_status()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_deterministic_and_empty_grid():
    H, W, heads = 9, 16, 2
    N = 4 * H * W
    q, k, v, g, dy = (si.normal(9710 + i, (1, N, heads * 128)).cuda() for i in range(5))
    rope = sana.Rope(4, H, W, (22, 21, 21))
    a = sana.linattn_bwd(q, k, v, g, rope, (4, H, W), heads, dy)
    b = sana.linattn_bwd(q, k, v, g, rope, (4, H, W), heads, dy)
    sana.sync_status()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    e = torch.empty(1, 0, heads * 128, dtype=torch.bfloat16, device="cuda")
    out = sana.linattn_bwd(e, e, e, None, rope, (0, H, W), heads, e)
    sana.sync_status()
    assert out[0].numel() == 0 and out[3] is None


def test_720p_sampled_rows_per_head():
    """The 720p/5s layer (24 heads, N = 75,600, gated): every head's gradients
    from the oracle (heads are independent), compared on sampled tokens."""
    wl = si.P720
    q, k, v, g = si.qkvg(wl)
    dy = si.normal(9720, (1, wl.N, wl.C))
    grid = (wl.T, wl.H, wl.W)
    rope = sana.Rope(wl.T, wl.H, wl.W, wl.rope_split)
    grads = sana.linattn_bwd(q.cuda(), k.cuda(), v.cuda(), g.cuda(), rope, grid, wl.heads,
                             dy.cuda())
    sana.sync_status()
    grads = [x.cpu() for x in grads]
    rows = np.unique(np.random.default_rng(12).choice(wl.N, size=256, replace=False))
    worst = 0.0
    for h in range(wl.heads):
        cols = slice(h * 128, (h + 1) * 128)
        ref = orc.linattn_backward(f64(q[:, :, cols]), f64(k[:, :, cols]), f64(v[:, :, cols]),
                                   grid, wl.rope_split, 1, f64(dy[:, :, cols]),
                                   gate=f64(g[:, :, cols]))
        for gg, rr in zip(grads, ref):
            e = orc.max_rel_err(f64(gg[:, rows, cols]), rr[:, rows])
            worst = max(worst, e)
            assert e <= BF16_TOL, (h, e)
