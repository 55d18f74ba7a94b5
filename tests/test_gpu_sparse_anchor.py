"""GPU parity of the block-sparse softmax anchor (sana_softmax_anchor_sparse_fwd).

Attention over a given tile list is compared with the float64 oracle on the
same list (lists made by the oracle or by the test, never by the GPU).  The
GPU's own tile selection is checked for validity against the oracle's pooled
scores: every kept tile must score at least as high as every dropped tile, up
to a tolerance for the bf16 rounding of the rotated operands."""

import numpy as np
import pytest
import torch

import sana_inputs as si
from oracle import sana_oracle as orc
from tests._sana import sana

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
SPLIT = (22, 21, 21)


def f64(t):
    return si.as_f64(t)


def inputs(seed, B, N, heads):
    return tuple(si.normal(seed + i, (B, N, heads * 128)) for i in range(4))


def check_selection(tiles, scores, keep):
    """tiles [B, h, nqb, keep] from the GPU; scores [B, h, nqb, nkt] from the oracle."""
    nkt = scores.shape[-1]
    for idx in np.ndindex(*tiles.shape[:-1]):
        sel = tiles[idx]
        assert np.all(np.diff(sel) > 0), (idx, sel)          # ascending, distinct
        assert sel[0] >= 0 and sel[-1] < nkt, (idx, sel)
        row = scores[idx]
        if keep == nkt:
            continue
        dropped = np.setdiff1d(np.arange(nkt), sel)
        tol = 1e-2 * (row.max() - row.min())
        assert row[sel].min() >= row[dropped].max() - tol, (idx, row[sel].min(), row[dropped].max())


def test_all_tiles_kept_equals_the_dense_anchor():
    H, W, heads = 7, 19, 2
    T = 6
    N = T * H * W  # 798 tokens: 7 key tiles, 4 query blocks, ragged tails
    q, k, v, g = (t.cuda() for t in inputs(9600, 2, N, heads))
    rope = sana.Rope(T, H, W, SPLIT)
    nkt = sana.anchor_tile_count(N)
    y, tiles = sana.softmax_anchor_sparse_fwd(q, k, v, g, rope, (T, H, W), heads, nkt)
    yd = sana.softmax_anchor_fwd(q, k, v, g, rope, (T, H, W), heads)
    sana.sync_status()
    assert torch.equal(tiles.cpu(), torch.arange(nkt, dtype=torch.int32).expand_as(tiles.cpu()))
    assert orc.max_rel_err(f64(y.cpu()), f64(yd.cpu())) <= 1e-5


@pytest.mark.parametrize("keep", [1, 3, 5])
def test_given_tile_lists_match_the_oracle(keep):
    """Random distinct tile lists per (batch, head, block), in arbitrary order."""
    H, W, heads = 7, 19, 2
    T = 6
    N = T * H * W
    B = 2
    q, k, v, g = inputs(9610, B, N, heads)
    nkt = sana.anchor_tile_count(N)
    nqb = (nkt + 1) // 2
    rng = np.random.default_rng(keep)
    lists = np.stack([rng.permutation(nkt)[:keep] for _ in range(B * heads * nqb)])
    lists = lists.reshape(B, heads, nqb, keep)
    rope = sana.Rope(T, H, W, SPLIT)
    tiles = torch.tensor(lists, dtype=torch.int32, device="cuda")
    y, _ = sana.softmax_anchor_sparse_fwd(q.cuda(), k.cuda(), v.cuda(), g.cuda(), rope, (T, H, W),
                                          heads, keep, tiles=tiles, select=False)
    sana.sync_status()
    assert torch.equal(tiles.cpu(), torch.tensor(lists, dtype=torch.int32))  # left as given
    yo = orc.softmax_anchor_tiles(f64(q), f64(k), f64(v), (T, H, W), SPLIT, heads, lists,
                                  gate=f64(g))
    assert orc.max_rel_err(f64(y.cpu()), yo) <= BF16_TOL


def test_library_selection_is_valid_and_its_output_matches_the_oracle():
    H, W, heads = 9, 16, 2
    T = 14
    N = T * H * W  # 2016 tokens: 16 key tiles, 8 query blocks
    q, k, v, g = inputs(9620, 1, N, heads)
    nkt = sana.anchor_tile_count(N)
    keep = 4
    rope = sana.Rope(T, H, W, SPLIT)
    y, tiles = sana.softmax_anchor_sparse_fwd(q.cuda(), k.cuda(), v.cuda(), g.cuda(), rope,
                                              (T, H, W), heads, keep)
    sana.sync_status()
    scores = orc.anchor_block_scores(f64(q), f64(k), (T, H, W), SPLIT, heads)
    check_selection(tiles.cpu().numpy(), scores, keep)
    # the output for the oracle's own selection, where it agrees with the GPU's
    mine = orc.anchor_block_select(scores, keep)
    same = np.all(mine == tiles.cpu().numpy(), axis=-1)
    assert same.mean() > 0.9
    yo = orc.softmax_anchor_tiles(f64(q), f64(k), f64(v), (T, H, W), SPLIT, heads, mine,
                                  gate=f64(g))
    yg = f64(y.cpu())
    for h in range(heads):
        for qb in range(mine.shape[2]):
            if not same[0, h, qb]:
                continue
            rows = slice(qb * 256, min(N, (qb + 1) * 256))
            cols = slice(h * 128, (h + 1) * 128)
            assert orc.max_rel_err(yg[:, rows, cols], yo[:, rows, cols]) <= BF16_TOL, (h, qb)


def test_720p_quarter_density_sampled():
    """720p/5s, 24 heads, 148 of 591 key tiles per block (25%): an oracle-made
    list through the kernel on sampled rows, and the library's own selection
    checked against the oracle's pooled scores."""
    wl = si.P720
    q, k, v, g = si.qkvg(wl)
    grid = (wl.T, wl.H, wl.W)
    nkt = sana.anchor_tile_count(wl.N)
    keep = (nkt + 3) // 4
    scores = orc.anchor_block_scores(f64(q), f64(k), grid, wl.rope_split, wl.heads)
    mine = orc.anchor_block_select(scores, keep)
    rope = sana.Rope(wl.T, wl.H, wl.W, wl.rope_split)
    qc, kc, vc, gc = q.cuda(), k.cuda(), v.cuda(), g.cuda()
    y, _ = sana.softmax_anchor_sparse_fwd(qc, kc, vc, gc, rope, grid, wl.heads, keep,
                                          tiles=torch.tensor(mine, dtype=torch.int32, device="cuda"),
                                          select=False)
    sana.sync_status()
    rows = np.unique(np.random.default_rng(11).choice(wl.N, size=24, replace=False))
    yo = orc.softmax_anchor_tiles(f64(q), f64(k), f64(v), grid, wl.rope_split, wl.heads, mine,
                                  gate=f64(g), rows=rows)
    assert orc.max_rel_err(f64(y.cpu()[:, rows]), yo) <= BF16_TOL
    _, tiles = sana.softmax_anchor_sparse_fwd(qc, kc, vc, gc, rope, grid, wl.heads, keep)
    sana.sync_status()
    check_selection(tiles.cpu().numpy(), scores, keep)
