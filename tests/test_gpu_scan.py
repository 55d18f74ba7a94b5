"""GPU parity of the whole-sequence block-causal entry point
(sana_linattn_block_causal_scan) against the float64 oracle's block sequence.

Bars as for the other linear-attention paths: max relative error <= 1e-4 for
fp32 and <= 2e-2 for bf16, on outputs and on the committed state."""

import numpy as np
import pytest
import torch

import sana_inputs as si
from oracle import sana_oracle as orc
from tests._sana import sana

pytestmark = pytest.mark.gpu

F32_TOL = 1e-4
BF16_TOL = 2e-2


def f64(t):
    return si.as_f64(t)


def run_both(q, k, v, g, grid, frames, t_offset, split, heads, S0, z0, tol, commit=True,
             t_total=None):
    T, H, W = grid
    B, N, C = q.shape
    D = C // heads
    rope = sana.Rope(t_total or t_offset + T, H, W, split)
    S = torch.tensor(S0, dtype=torch.float32, device="cuda")
    z = torch.tensor(z0, dtype=torch.float32, device="cuda")
    y = sana.linattn_block_causal_scan(q.cuda(), k.cuda(), v.cuda(), None if g is None else g.cuda(),
                                       rope, grid, t_offset, heads, frames, S, z, commit=commit)
    sana.sync_status()
    yo, So, zo = orc.linattn_block_causal_sequence(
        f64(q), f64(k), f64(v), grid, frames, t_offset, split, heads, S0, z0,
        gate=None if g is None else f64(g), commit=commit)
    e = (orc.max_rel_err(f64(y), yo), orc.max_rel_err(S.cpu().numpy().astype(np.float64), So),
         orc.max_rel_err(z.cpu().numpy().astype(np.float64), zo))
    assert max(e) <= tol, e
    return y, S, z


@pytest.mark.parametrize("frames", [1, 2, 3, 7, 9])
def test_fp32_tiny_every_block_length(frames):
    """7 frames of 4 x 4 in blocks of 1, 2 (3 + remainder), 3, 7 and 9 (one block)."""
    H, W, heads, D = 4, 4, 2, 16
    T = 7
    N = T * H * W
    q, k, v, g = (si.normal(9500 + i, (1, N, heads * D), torch.float32) for i in range(4))
    z0 = np.zeros((1, heads, D))
    S0 = np.zeros((1, heads, D, D))
    run_both(q, k, v, g, (T, H, W), frames, 0, (2, 3, 3), heads, S0, z0, F32_TOL)


def test_fp32_from_a_carried_state_with_frame_offset():
    H, W, heads, D = 3, 5, 3, 32
    T = 5
    N = T * H * W
    q, k, v, g = (si.normal(9510 + i, (2, N, heads * D), torch.float32) for i in range(4))
    rng = np.random.default_rng(9)
    S0 = np.abs(rng.standard_normal((2, heads, D, D))) * 3
    z0 = np.abs(rng.standard_normal((2, heads, D))) * 3
    S0 = S0.astype(np.float32).astype(np.float64)
    z0 = z0.astype(np.float32).astype(np.float64)
    run_both(q, k, v, g, (T, H, W), 2, 4, (6, 5, 5), heads, S0, z0, F32_TOL, t_total=9)


@pytest.mark.parametrize("B,frames,grid", [(2, 3, (9, 9, 16)), (1, 2, (9, 9, 16)),
                                           (2, 4, (9, 9, 16)), (1, 5, (6, 7, 19))])
def test_bf16_ragged_blocks(B, frames, grid):
    """Blocks of 432 / 288 / 576 / 665 tokens (ragged against 128-token tiles),
    with and without a short last block."""
    heads, D = 2, 128
    T, H, W = grid
    N = T * H * W
    q, k, v, g = (si.normal(9520 + i, (B, N, heads * D)) for i in range(4))
    S0 = np.zeros((B, heads, D, D))
    z0 = np.zeros((B, heads, D))
    run_both(q, k, v, g, grid, frames, 0, (22, 21, 21), heads, S0, z0, BF16_TOL)


def test_bf16_commit_flag_and_agreement_with_block_steps():
    """commit=0 keeps the state and gives the commit=1 output; the sequence
    equals block-by-block steps on the same device (to bf16 rounding)."""
    H, W, heads, D = 9, 16, 2, 128
    T, frames = 8, 3
    N = T * H * W
    hw = H * W
    q, k, v, g = (si.normal(9530 + i, (1, N, heads * D)).cuda() for i in range(4))
    rope = sana.Rope(T + 2, H, W, (22, 21, 21))
    S = torch.randn(1, heads, D, D, device="cuda").abs()
    z = torch.randn(1, heads, D, device="cuda").abs() * 10
    S0, z0 = S.clone(), z.clone()
    y_nc = sana.linattn_block_causal_scan(q, k, v, g, rope, (T, H, W), 2, heads, frames, S, z,
                                          commit=False)
    sana.sync_status()
    assert torch.equal(S, S0) and torch.equal(z, z0)
    y_c = sana.linattn_block_causal_scan(q, k, v, g, rope, (T, H, W), 2, heads, frames, S, z,
                                         commit=True)
    sana.sync_status()
    assert torch.equal(y_nc, y_c)
    S2, z2 = S0.clone(), z0.clone()
    ys = []
    for t0 in range(0, T, frames):
        f = min(frames, T - t0)
        sl = slice(t0 * hw, (t0 + f) * hw)
        ys.append(sana.linattn_block_causal_step(q[:, sl], k[:, sl], v[:, sl], g[:, sl], rope,
                                                 (f, H, W), 2 + t0, heads, S2, z2))
    sana.sync_status()
    y_steps = torch.cat(ys, dim=1)
    assert orc.max_rel_err(f64(y_c.cpu()), f64(y_steps.cpu())) <= 1e-2
    assert orc.max_rel_err(S.cpu().double().numpy(), S2.cpu().double().numpy()) <= 1e-5
    assert orc.max_rel_err(z.cpu().double().numpy(), z2.cpu().double().numpy()) <= 1e-5


def test_empty_sequence_is_a_no_op_and_bad_block_length_is_rejected():
    H, W, heads, D = 4, 4, 2, 128
    rope = sana.Rope(4, H, W, (22, 21, 21))
    e = torch.empty(1, 0, heads * D, dtype=torch.bfloat16, device="cuda")
    S = torch.ones(1, heads, D, D, device="cuda")
    z = torch.ones(1, heads, D, device="cuda")
    y = sana.linattn_block_causal_scan(e, e, e, None, rope, (0, H, W), 0, heads, 3, S, z)
    sana.sync_status()
    assert y.numel() == 0 and bool((S == 1).all()) and bool((z == 1).all())
    q = torch.zeros(1, 2 * H * W, heads * D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sana.SanaError):
        sana.linattn_block_causal_scan(q, q, q, None, rope, (2, H, W), 0, heads, 0, S, z)


def test_720p_ten_frames_sampled():
    """10 frames of the 720p grid (36,000 tokens, 24 heads) in blocks of 3
    frames plus a 1-frame block: the committed state in full, outputs on
    sampled tokens of every block."""
    wl = si.LONG
    H, W, heads, D = wl.H, wl.W, wl.heads, wl.D
    T, frames = 10, 3
    hw = H * W
    N = T * hw
    q, k, v = (si.normal(9540 + i, (1, N, heads * D)) for i in range(3))
    rope = sana.Rope(T, H, W, wl.rope_split)
    S = torch.zeros(1, heads, D, D, device="cuda")
    z = torch.zeros(1, heads, D, device="cuda")
    y = sana.linattn_block_causal_scan(q.cuda(), k.cuda(), v.cuda(), None, rope, (T, H, W), 0,
                                       heads, frames, S, z)
    sana.sync_status()
    y = y.cpu()
    So = np.zeros((1, heads, D, D))
    zo = np.zeros((1, heads, D))
    rng = np.random.default_rng(10)
    for t0 in range(0, T, frames):
        f = min(frames, T - t0)
        sl = slice(t0 * hw, (t0 + f) * hw)
        ang = orc.rope_angles(f, H, W, *wl.rope_split, t_offset=t0)
        Sc, zc = orc.linattn_state(f64(k[:, sl]), f64(v[:, sl]), ang, heads)
        So, zo = So + Sc, zo + zc
        rows = np.unique(rng.choice(f * hw, size=48, replace=False))
        yo = orc.linattn_apply(f64(q[:, sl][:, rows]), So, zo, ang[rows], heads)
        assert orc.max_rel_err(f64(y[:, sl][:, rows]), yo) <= BF16_TOL, t0
    assert orc.max_rel_err(S.cpu().double().numpy(), So) <= BF16_TOL
    assert orc.max_rel_err(z.cpu().double().numpy(), zo) <= BF16_TOL
