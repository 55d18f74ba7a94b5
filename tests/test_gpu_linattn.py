"""GPU parity of the linear-attention entry points against the float64 oracle.

Bars: max relative error (max |gpu - oracle| / max |oracle|) <= 1e-4 for
fp32 and <= 2e-2 for bf16, on outputs and on the carried causal state."""

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


def gpu_lin(q, k, v, g, grid, split, heads, t_total=None):
    rope = sana.Rope(t_total or grid[0], grid[1], grid[2], split)
    y = sana.linattn_fwd(q.cuda(), k.cuda(), v.cuda(), None if g is None else g.cuda(), rope,
                         grid, heads)
    sana.sync_status()
    return y


def test_tiny_fp32_config():
    wl = si.TINY
    q, k, v, g = si.qkvg(wl)
    grid = (wl.T, wl.H, wl.W)
    y = gpu_lin(q, k, v, g, grid, wl.rope_split, wl.heads).cpu()
    yo, _, _ = orc.linattn_bidirectional(f64(q), f64(k), f64(v), grid, wl.rope_split, wl.heads,
                                         gate=f64(g))
    assert orc.max_rel_err(f64(y), yo) <= F32_TOL
    # ungated
    y = gpu_lin(q, k, v, None, grid, wl.rope_split, wl.heads).cpu()
    yo, _, _ = orc.linattn_bidirectional(f64(q), f64(k), f64(v), grid, wl.rope_split, wl.heads)
    assert orc.max_rel_err(f64(y), yo) <= F32_TOL


@pytest.mark.parametrize("D,heads,grid,split", [(32, 3, (3, 5, 7), (6, 5, 5)),
                                                (64, 2, (2, 9, 11), (10, 11, 11)),
                                                (128, 2, (1, 7, 19), (22, 21, 21))])
def test_fp32_other_head_dims(D, heads, grid, split):
    N = grid[0] * grid[1] * grid[2]
    q, k, v, g = (si.normal(7000 + i, (2, N, heads * D), torch.float32) for i in range(4))
    y = gpu_lin(q, k, v, g, grid, split, heads).cpu()
    yo, _, _ = orc.linattn_bidirectional(f64(q), f64(k), f64(v), grid, split, heads, gate=f64(g))
    assert orc.max_rel_err(f64(y), yo) <= F32_TOL


@pytest.mark.parametrize("B,heads,grid", [(1, 2, (2, 4, 4)),     # N = 32: one partial tile
                                          (2, 3, (3, 5, 9)),     # N = 135: ragged tail of 7
                                          (1, 1, (1, 1, 1)),     # a single token
                                          (1, 4, (5, 16, 16)),   # N = 1280: 10 full tiles
                                          (2, 2, (7, 13, 17))])  # N = 1547, several splits
def test_bf16_small_with_ragged_tails(B, heads, grid):
    N = grid[0] * grid[1] * grid[2]
    C = heads * 128
    q, k, v, g = (si.normal(8000 + 10 * N + i, (B, N, C)) for i in range(4))
    split = (22, 21, 21)
    y = gpu_lin(q, k, v, g, grid, split, heads).cpu()
    yo, _, _ = orc.linattn_bidirectional(f64(q), f64(k), f64(v), grid, split, heads, gate=f64(g))
    assert orc.max_rel_err(f64(y), yo) <= BF16_TOL
    y = gpu_lin(q, k, v, None, grid, split, heads).cpu()
    yo, _, _ = orc.linattn_bidirectional(f64(q), f64(k), f64(v), grid, split, heads)
    assert orc.max_rel_err(f64(y), yo) <= BF16_TOL


@pytest.mark.parametrize("gated", [True, False])
def test_two_phases_equal_the_fused_layer(gated):
    """sana_linattn_state then sana_linattn_apply (the standalone output pass,
    which loads nothing before its launch dependency resolves) give the fused
    layer's output bit for bit, and the state (S, z) matches the oracle's."""
    B, heads, grid = 2, 2, (3, 9, 16)
    N = grid[0] * grid[1] * grid[2]
    q, k, v, g = (si.normal(10900 + i, (B, N, heads * 128)) for i in range(4))
    if not gated:
        g = None
    rope = sana.Rope(*grid, (22, 21, 21))
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    gc = None if g is None else g.cuda()
    y1 = sana.linattn_fwd(qc, kc, vc, gc, rope, grid, heads)
    S, z = sana.linattn_state(kc, vc, rope, grid, heads)
    y2 = sana.linattn_apply(qc, gc, rope, grid, heads, S, z)
    sana.sync_status()
    assert torch.equal(y1, y2)
    ang = orc.rope_angles(*grid, 22, 21, 21)
    So, zo = orc.linattn_state(f64(k), f64(v), ang, heads)
    assert orc.max_rel_err(S.cpu().double().numpy(), So) <= BF16_TOL
    assert orc.max_rel_err(z.cpu().double().numpy(), zo) <= BF16_TOL
    yo, _, _ = orc.linattn_bidirectional(f64(q), f64(k), f64(v), grid, (22, 21, 21), heads,
                                         gate=None if g is None else f64(g))
    assert orc.max_rel_err(f64(y2), yo) <= BF16_TOL


def test_empty_grid_is_a_no_op():
    rope = sana.Rope(1, 4, 4, (22, 21, 21))
    q = torch.zeros(1, 0, 256, dtype=torch.bfloat16, device="cuda")
    y = sana.linattn_fwd(q, q.clone(), q.clone(), None, rope, (0, 4, 4), 2)
    sana.sync_status()
    assert y.shape == (1, 0, 256)


def sampled_rows(N, count, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([rng.choice(N, size=min(count, N), replace=False),
                                     np.arange(max(0, N - 80), N), [0]]))
    return rows


def full_size_sampled_check(wl, rows_count=768):
    """All heads, sampled tokens (plus the ragged tail) against the oracle,
    in the launch configuration the benchmark times."""
    q, k, v, g = si.qkvg(wl)
    grid = (wl.T, wl.H, wl.W)
    y = gpu_lin(q, k, v, g, grid, wl.rope_split, wl.heads)
    y2 = gpu_lin(q, k, v, g, grid, wl.rope_split, wl.heads)
    assert torch.equal(y, y2), "results are not bit-reproducible"
    y = y.cpu()
    ang = orc.rope_angles(*grid, *wl.rope_split)
    rows = sampled_rows(wl.N, rows_count, wl.config)
    D = wl.D
    got, ref = [], []
    for h in range(wl.heads):
        sl = slice(h * D, (h + 1) * D)
        S, z = orc.linattn_state(f64(k[:, :, sl]), f64(v[:, :, sl]), ang, 1)
        ref.append(orc.linattn_apply(f64(q[:, rows, sl]), S, z, ang[rows], 1, gate=f64(g[:, rows, sl])))
        got.append(f64(y[:, rows, sl]))
    err = orc.max_rel_err(np.concatenate(got, -1), np.concatenate(ref, -1))
    assert err <= BF16_TOL, err
    return err


@pytest.mark.parametrize("c", [-12.0, -8.0, -4.0, 6.0])
def test_gate_accuracy_at_saturated_logits(c):
    """Every gate logit equal to c: the output is sigmoid(c) times the ungated
    layer.  The gate's tanh form has an absolute error of about 2.5e-4, so for
    c >= -4 (sigmoid(c) >= 0.018) the parity measure of the gated output holds;
    further out the output is under 2% of the ungated one and only its error
    relative to the ungated output's scale is bounded (here by 1e-3)."""
    grid, heads = (3, 8, 16), 2
    N, C = 384, 256
    q, k, v = (si.normal(7600 + i, (1, N, C)) for i in range(3))
    g = torch.full((1, N, C), c, dtype=torch.bfloat16)
    y = gpu_lin(q, k, v, g, grid, (22, 21, 21), heads).cpu()
    yo, _, _ = orc.linattn_bidirectional(f64(q), f64(k), f64(v), grid, (22, 21, 21), heads,
                                         gate=f64(g))
    if c >= -4.0:
        err = orc.max_rel_err(f64(y), yo)
        assert err <= BF16_TOL, err
    else:
        ungated, _, _ = orc.linattn_bidirectional(f64(q), f64(k), f64(v), grid, (22, 21, 21),
                                                  heads)
        err = np.max(np.abs(f64(y) - yo)) / np.max(np.abs(ungated))
        assert err <= 1e-3, err


def test_480p_full_size_sampled():
    full_size_sampled_check(si.P480)


def test_720p_full_size_sampled():
    full_size_sampled_check(si.P720)


# ---------------------------------------------------------------- block-causal

def run_causal(wl_like, chunks, q, k, v, g, dtype_tol, B, heads, D, H, W, split, check_every=True,
               rows=None):
    """Run chunks through the GPU step and the oracle; compare outputs and state."""
    T_total = sum(f for _, f in chunks)
    rope = sana.Rope(T_total, H, W, split)
    S = torch.zeros(B, heads, D, D, dtype=torch.float32, device="cuda")
    z = torch.zeros(B, heads, D, dtype=torch.float32, device="cuda")
    So = np.zeros((B, heads, D, D))
    zo = np.zeros((B, heads, D))
    worst = 0.0
    for ci, (t0, f) in enumerate(chunks):
        sl = slice(t0 * H * W, (t0 + f) * H * W)
        qc, kc, vc = q[:, sl], k[:, sl], v[:, sl]
        gc = None if g is None else g[:, sl]
        y = sana.linattn_block_causal_step(qc.cuda(), kc.cuda(), vc.cuda(),
                                           None if gc is None else gc.cuda(), rope, (f, H, W), t0,
                                           heads, S, z, commit=True)
        sana.sync_status()
        yo, So, zo = orc.linattn_block_causal_step(f64(qc), f64(kc), f64(vc), (f, H, W), t0, split,
                                                   heads, So, zo, gate=None if gc is None else f64(gc))
        e = max(orc.max_rel_err(f64(y), yo), orc.max_rel_err(S.cpu().numpy(), So),
                orc.max_rel_err(z.cpu().numpy(), zo))
        worst = max(worst, e)
        assert e <= dtype_tol, (ci, e)
    return worst


@pytest.mark.parametrize("chunk_frames", [[1, 1], [2, 1, 3], [6]])
def test_causal_fp32_tiny(chunk_frames):
    wl = si.TINY
    H, W, heads, D = 4, 4, 2, 16
    T = sum(chunk_frames)
    N = T * H * W
    q, k, v, g = (si.normal(9000 + i, (1, N, heads * D), torch.float32) for i in range(4))
    chunks, t0 = [], 0
    for f in chunk_frames:
        chunks.append((t0, f))
        t0 += f
    run_causal(wl, chunks, q, k, v, g, F32_TOL, 1, heads, D, H, W, wl.rope_split)


def test_causal_bf16_multi_chunk_and_commit_flag():
    H, W, heads, D = 9, 16, 2, 128
    split = (22, 21, 21)
    chunks = [(0, 3), (3, 3), (6, 2), (8, 1)]
    N = 9 * H * W
    q, k, v, g = (si.normal(9100 + i, (2, N, heads * D)) for i in range(4))
    run_causal(None, chunks, q, k, v, g, BF16_TOL, 2, heads, D, H, W, split)
    # commit = 0 leaves the state untouched and gives the same output as commit = 1
    rope = sana.Rope(9, H, W, split)
    S = torch.randn(2, heads, D, D, device="cuda").abs()
    z = torch.randn(2, heads, D, device="cuda").abs()
    S0, z0 = S.clone(), z.clone()
    sl = slice(3 * H * W, 6 * H * W)
    args = (q[:, sl].cuda(), k[:, sl].cuda(), v[:, sl].cuda(), g[:, sl].cuda(), rope, (3, H, W), 3,
            heads)
    y_nc = sana.linattn_block_causal_step(*args, S, z, commit=False)
    sana.sync_status()
    assert torch.equal(S, S0) and torch.equal(z, z0)
    y_c = sana.linattn_block_causal_step(*args, S, z, commit=True)
    sana.sync_status()
    assert torch.equal(y_nc, y_c)
    assert not torch.equal(S, S0)


def test_causal_state_checkpoint_restore_is_bit_exact(tmp_path):
    H, W, heads, D = 6, 10, 2, 128
    split = (22, 21, 21)
    N = 4 * H * W
    q, k, v = (si.normal(9200 + i, (1, N, heads * D)).cuda() for i in range(3))
    rope = sana.Rope(4, H, W, split)
    S = torch.zeros(1, heads, D, D, device="cuda")
    z = torch.zeros(1, heads, D, device="cuda")
    hw = H * W
    sana.linattn_block_causal_step(q[:, :2 * hw], k[:, :2 * hw], v[:, :2 * hw], None, rope,
                                   (2, H, W), 0, heads, S, z)
    torch.save({"S": S.cpu(), "z": z.cpu()}, tmp_path / "state.pt")
    y_a = sana.linattn_block_causal_step(q[:, 2 * hw:], k[:, 2 * hw:], v[:, 2 * hw:], None, rope,
                                         (2, H, W), 2, heads, S, z)
    st = torch.load(tmp_path / "state.pt")
    S2, z2 = st["S"].cuda(), st["z"].cuda()
    y_b = sana.linattn_block_causal_step(q[:, 2 * hw:], k[:, 2 * hw:], v[:, 2 * hw:], None, rope,
                                         (2, H, W), 2, heads, S2, z2)
    sana.sync_status()
    assert torch.equal(y_a, y_b) and torch.equal(S, S2) and torch.equal(z, z2)


@pytest.mark.slow
def test_causal_720p_60s_full_run():
    """All 81 chunks (80 x 3 frames + 1) of the 720p/60s workload; outputs on
    sampled tokens and the full state after every chunk."""
    wl = si.LONG
    H, W, heads, D = wl.H, wl.W, wl.heads, wl.D
    rope = sana.Rope(wl.T, H, W, wl.rope_split)
    S = torch.zeros(wl.B, heads, D, D, device="cuda")
    z = torch.zeros(wl.B, heads, D, device="cuda")
    So = np.zeros((wl.B, heads, D, D))
    zo = np.zeros((wl.B, heads, D))
    ws = torch.empty(sana.linattn_workspace_size(wl.B, (3, H, W), heads, D, 1), dtype=torch.uint8,
                     device="cuda")
    rng = np.random.default_rng(4)
    for ci, (t0, f) in enumerate(si.chunk_frames(wl)):
        q, k, v = si.causal_chunk(wl, ci, f)
        y = sana.linattn_block_causal_step(q.cuda(), k.cuda(), v.cuda(), None, rope, (f, H, W), t0,
                                           heads, S, z, ws=ws)
        sana.sync_status()
        ang = orc.rope_angles(f, H, W, *wl.rope_split, t_offset=t0)
        Sc, zc = orc.linattn_state(f64(k), f64(v), ang, heads)
        So, zo = So + Sc, zo + zc
        rows = np.unique(rng.choice(f * H * W, size=64, replace=False))
        yo = orc.linattn_apply(f64(q[:, rows]), So, zo, ang[rows], heads)
        e = max(orc.max_rel_err(f64(y[:, rows]), yo), orc.max_rel_err(S.cpu().numpy(), So),
                orc.max_rel_err(z.cpu().numpy(), zo))
        assert e <= BF16_TOL, (ci, e)


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    """A wait that can never complete gives up after its limit, the host reads
    SANA_ERR_TIMEOUT from the device status word, and later calls work."""
    from softmax_attention_sana_b200 import _lib as L
    sana._lib.selftest_bounded_wait(50)
    with pytest.raises(L.SanaError) as e:
        sana.sync_status()
    assert e.value.status == L.SANA_ERR_TIMEOUT
    sana.sync_status()  # the status word was cleared
    wl = si.TINY
    q, k, v, g = si.qkvg(wl)
    y = gpu_lin(q, k, v, g, (wl.T, wl.H, wl.W), wl.rope_split, wl.heads).cpu()
    yo, _, _ = orc.linattn_bidirectional(f64(q), f64(k), f64(v), (wl.T, wl.H, wl.W),
                                         wl.rope_split, wl.heads, gate=f64(g))
    assert orc.max_rel_err(f64(y), yo) <= F32_TOL
