"""GPU parity of the AttnRes router, RMSNorm, the projection GEMM and the
hybrid stack against the float64 oracle."""

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


# ---------------------------------------------------------------- AttnRes router

@pytest.mark.parametrize("S,B,N,C", [(1, 1, 40, 256), (2, 2, 33, 512), (3, 1, 257, 3072),
                                     (5, 1, 64, 1024), (16, 1, 17, 512)])
def test_attnres_route_bf16(S, B, N, C):
    srcs = [si.normal(12000 + 37 * S + i, (B, N, C)) for i in range(S)]
    w = si.normal(12100 + S, (C,), torch.float32, C ** -0.5)
    h, alpha = sana.attnres_route([x.cuda() for x in srcs], w.cuda(), want_alpha=True)
    sana.sync_status()
    ho, ao = orc.attnres_route([f64(x) for x in srcs], f64(w))
    assert orc.max_rel_err(f64(h), ho) <= BF16_TOL
    assert np.max(np.abs(alpha.cpu().numpy() - ao)) <= 1e-4
    np.testing.assert_allclose(alpha.sum(-1).cpu().numpy(), 1.0, rtol=1e-5)
    if S == 1:
        assert torch.equal(h.cpu(), srcs[0])


def test_attnres_route_fp32():
    srcs = [si.normal(12200 + i, (1, 50, 256), torch.float32) for i in range(3)]
    w = si.normal(12210, (256,), torch.float32, 256 ** -0.5)
    h = sana.attnres_route([x.cuda() for x in srcs], w.cuda())
    sana.sync_status()
    ho, _ = orc.attnres_route([f64(x) for x in srcs], f64(w))
    assert orc.max_rel_err(f64(h), ho) <= F32_TOL


def test_attnres_route_720p_three_sources():
    N, C = si.P720.N, si.P720.C
    srcs = si.attnres_sources(5, 3, 1, N, C)
    w_attn, _ = si.router_queries(5, C)
    h = sana.attnres_route([x.cuda() for x in srcs], w_attn.cuda())
    sana.sync_status()
    rows = np.unique(np.random.default_rng(5).choice(N, 2048, replace=False))
    ho, _ = orc.attnres_route([f64(x[:, rows]) for x in srcs], f64(w_attn))
    assert orc.max_rel_err(f64(h[:, rows]), ho) <= BF16_TOL


def test_rmsnorm():
    x = si.normal(12300, (3, 77, 3072))
    y = sana.rmsnorm(x.cuda())
    sana.sync_status()
    assert orc.max_rel_err(f64(y), orc.rmsnorm(f64(x))) <= BF16_TOL
    x = si.normal(12301, (5, 256), torch.float32)
    y = sana.rmsnorm(x.cuda())
    sana.sync_status()
    assert orc.max_rel_err(f64(y), orc.rmsnorm(f64(x))) <= F32_TOL


# ---------------------------------------------------------------- GEMM

@pytest.mark.parametrize("M,N,K", [(300, 512, 256), (128, 256, 64), (1, 48, 128),
                                   (1000, 768, 1024), (77, 4096, 512)])
def test_gemm_epilogues(M, N, K):
    A = si.normal(12400 + M, (M, K))
    W = si.normal(12500 + N, (N, K), scale=K ** -0.5)
    ref = f64(A) @ f64(W).T
    y = sana.gemm_bf16(A.cuda(), W.cuda())
    sana.sync_status()
    assert orc.max_rel_err(f64(y), ref) <= BF16_TOL
    y = sana.gemm_bf16(A.cuda(), W.cuda(), epilogue=sana.EPI_SILU)
    sana.sync_status()
    assert orc.max_rel_err(f64(y), orc.silu(ref)) <= BF16_TOL
    base = si.normal(12600 + M, (M, N))
    y = base.cuda().clone()
    sana.gemm_bf16(A.cuda(), W.cuda(), out=y, epilogue=sana.EPI_RESIDUAL)
    sana.sync_status()
    assert orc.max_rel_err(f64(y), f64(base) + ref) <= BF16_TOL


def test_gemm_720p_qkvg_projection_sampled_rows():
    """The stack's largest projection: (75,600 x 3072) . (12,288 x 3072)^T."""
    M, C = si.P720.N, si.P720.C
    A = si.normal(12700, (M, C))
    W = si.normal(12701, (4 * C, C), scale=C ** -0.5)
    y = sana.gemm_bf16(A.cuda(), W.cuda())
    sana.sync_status()
    rows = np.unique(np.concatenate([np.random.default_rng(7).choice(M, 512, replace=False),
                                     np.arange(M - 40, M)]))
    ref = f64(A[rows]) @ f64(W).T
    assert orc.max_rel_err(f64(y[rows]), ref) <= BF16_TOL


# ---------------------------------------------------------------- stack

def _stack_inputs(C, N, layers, ffn_mult, seed):
    x = si.normal(seed, (1, N, C))
    ws = si.projection_weights(seed // 1000, layers, C, ffn_mult)
    w_attn, w_ffn = si.router_queries(seed // 1000, C)
    return x, ws, w_attn, w_ffn


def _run_stack(x, ws, w_attn, w_ffn, grid, heads, cfg):
    rope = sana.Rope(grid[0], grid[1], grid[2], (22, 21, 21))
    wsd = [{k: v.cuda() for k, v in d.items()} for d in ws]
    y = sana.hybrid_stack_fwd(x.cuda(), wsd, w_attn.cuda(), w_ffn.cuda(), rope, grid, heads, cfg)
    sana.sync_status()
    return y


def _oracle_stack(x, ws, w_attn, w_ffn, grid, heads, layers, span, attnres, ffn, keep=0):
    wo = [{k: f64(v) for k, v in d.items()} for d in ws]
    return orc.hybrid_stack(f64(x), wo, f64(w_attn), f64(w_ffn), grid, (22, 21, 21), heads,
                            layers, block_span=span, use_attnres=attnres, ffn=ffn,
                            anchor_keep=keep)


@pytest.mark.parametrize("layers,span,attnres,ffn", [(4, 8, False, 0), (4, 8, False, 3),
                                                      (5, 2, True, 3), (8, 4, True, 0),
                                                      (16, 8, True, 3)])
def test_stack_small_against_oracle(layers, span, attnres, ffn):
    grid, heads = (2, 4, 8), 2
    C, N = 256, 64
    x, ws, w_attn, w_ffn = _stack_inputs(C, N, layers, ffn, 13000 + layers)
    cfg = sana.stack_config(layers, block_span=span, use_attnres=attnres, ffn_mult=ffn)
    y = _run_stack(x, ws, w_attn, w_ffn, grid, heads, cfg)
    yo = _oracle_stack(x, ws, w_attn, w_ffn, grid, heads, layers, span, attnres, ffn > 0)
    err = orc.max_rel_err(f64(y), yo)
    assert err <= BF16_TOL, err


@pytest.mark.parametrize("keep", [4, 2])
def test_stack_with_sparse_anchors_against_oracle(keep):
    """8 layers (2 anchors) on a 4 x 8 x 16 grid (512 tokens: 4 key tiles, 2
    query blocks): all 4 tiles kept (= dense anchors) and 2 of 4 kept."""
    grid, heads = (4, 8, 16), 2
    C, N = 256, 512
    layers, span = 8, 4
    x, ws, w_attn, w_ffn = _stack_inputs(C, N, layers, 3, 13100 + keep)
    cfg = sana.stack_config(layers, block_span=span, use_attnres=True, ffn_mult=3,
                            anchor_keep_tiles=keep)
    y = _run_stack(x, ws, w_attn, w_ffn, grid, heads, cfg)
    yo = _oracle_stack(x, ws, w_attn, w_ffn, grid, heads, layers, span, True, True, keep)
    err = orc.max_rel_err(f64(y), yo)
    assert err <= BF16_TOL, err


@pytest.mark.slow
@pytest.mark.parametrize("layers,attnres,ffn", [(4, False, 0), (16, True, 3)])
def test_stack_full_size_runs_deterministically(layers, attnres, ffn):
    """720p/5s group (4 layers, no AttnRes) and the 16-layer AttnRes stack:
    finite, bit-reproducible outputs.  (The float64 oracle cannot run these
    sizes; every stage is checked at full size by the tests above.)"""
    wl = si.STACK
    grid = (wl.T, wl.H, wl.W)
    x, ws, w_attn, w_ffn = _stack_inputs(wl.C, wl.N, layers, ffn, 5000 + layers)
    cfg = sana.stack_config(layers, block_span=8, use_attnres=attnres, ffn_mult=ffn)
    y1 = _run_stack(x, ws, w_attn, w_ffn, grid, wl.heads, cfg)
    y2 = _run_stack(x, ws, w_attn, w_ffn, grid, wl.heads, cfg)
    assert torch.isfinite(y1.float()).all()
    assert torch.equal(y1, y2)


@pytest.mark.slow
def test_stack_full_width_and_depth_short_sequence():
    """The 16-layer AttnRes stack at full width (24 heads x 128, hidden 3072,
    FFN 3C) on a 512-token grid, against the whole float64 oracle stack: the
    error accumulated over 32 sublayers of bf16 partial sums and residual
    routes, end to end."""
    grid, heads, layers = (2, 16, 16), 24, 16
    C, N = heads * 128, 512
    x, ws, w_attn, w_ffn = _stack_inputs(C, N, layers, 3, 15000 + layers)
    cfg = sana.stack_config(layers, block_span=8, use_attnres=True, ffn_mult=3)
    y = _run_stack(x, ws, w_attn, w_ffn, grid, heads, cfg)
    yo = _oracle_stack(x, ws, w_attn, w_ffn, grid, heads, layers, 8, True, True)
    err = orc.max_rel_err(f64(y), yo)
    print(f"16-layer stack, N=512, C=3072: max_rel {err:.3e} "
          f"elementwise {orc.elementwise_rel_err(f64(y), yo):.3e}")
    assert err <= BF16_TOL, err


def _mx_stack(x, ws, w_attn, w_ffn, grid, heads, cfg, wsd=None, ws_buf=None):
    rope = sana.Rope(grid[0], grid[1], grid[2], (22, 21, 21))
    if wsd is None:
        wsd = sana.mx_quantize_stack_weights([{k: v.cuda() for k, v in d.items()} for d in ws])
        for d in wsd:  # the MX form alone must suffice
            for key in ("qkvg", "o", "up", "down"):
                d.pop(key, None)
    y = sana.hybrid_stack_fwd(x.cuda(), wsd, w_attn.cuda(), w_ffn.cuda(), rope, grid, heads, cfg,
                              ws=ws_buf)
    sana.sync_status()
    return y, wsd


def test_stack_mx_projections_end_to_end():
    """Four layers without AttnRes or FFN, every projection as the MX projection
    (MXFP4 weights quantised by the library, activations quantised to MXFP8 on
    the fly), against the oracle stack with its MX option; C = 256 on a
    512-token grid.  (Deeper MX stacks are checked teacher-forced below: the
    quantiser is discontinuous, so a one-ulp bf16 difference upstream moves
    an element by a whole E4M3 step and the two sides drift apart with depth.)"""
    grid, heads, C, N, layers = (4, 8, 16), 2, 256, 512, 4
    x, ws, w_attn, w_ffn = _stack_inputs(C, N, layers, 0, 13204)
    cfg = sana.stack_config(layers, use_attnres=False, ffn_mult=0, mx_projections=True)
    y, _ = _mx_stack(x, ws, w_attn, w_ffn, grid, heads, cfg)
    wo = [{k: f64(v) for k, v in d.items()} for d in ws]
    yo = orc.hybrid_stack(f64(x), wo, f64(w_attn), f64(w_ffn), grid, (22, 21, 21), heads, layers,
                          use_attnres=False, ffn=False, mx=True)
    err = orc.max_rel_err(f64(y), yo)
    assert err <= BF16_TOL, err


def _bf16(a):
    return f64(torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16))


def test_stack_mx_projections_teacher_forced():
    """Eight layers with AttnRes (blocks of 4) and FFN 3C, MX projections,
    checked step by step on the GPU's own inputs of each step: the QKVG
    projection of the routed, normalised input (rounded to bf16 as the GPU
    stores it before quantising), W_o and the FFN projections of the GPU's
    attention output and FFN hidden state, and the partial sum."""
    grid, heads, C, N, layers, span = (4, 8, 16), 2, 256, 512, 8, 4
    x, ws, w_attn, w_ffn = _stack_inputs(C, N, layers, 3, 13208)
    wo = [{k: f64(v) for k, v in d.items()} for d in ws]
    cfg_for = lambda L: sana.stack_config(L, block_span=span, use_attnres=True, ffn_mult=3,
                                          mx_projections=True)
    buf = torch.empty(sana.hybrid_stack_workspace_size(1, grid, heads, cfg_for(layers)),
                      dtype=torch.uint8, device="cuda")
    wsd = None
    emb, summaries, partial = f64(x), [], None
    mx = orc.mx_linear
    for l in range(layers):
        cfg = cfg_for(l + 1)
        _, wsd = _mx_stack(x, ws, w_attn, w_ffn, grid, heads, cfg, wsd, buf)
        vw = sana.hybrid_stack_workspace_views(buf, 1, grid, heads, cfg)
        srcs = [emb] + summaries + ([partial] if partial is not None else [])
        h, _ = orc.attnres_route(srcs, f64(w_attn))
        xh = _bf16(orc.rmsnorm(h)[0])
        qkvg = mx(xh, wo[l]["qkvg"])
        for i, key in enumerate("qkvg"):
            err = orc.max_rel_err(f64(vw[key])[0], qkvg[:, i * C:(i + 1) * C])
            assert err <= BF16_TOL, (l, key, err)
        attn = f64(vw["attn"])[0]
        mid = _bf16(mx(attn, wo[l]["o"]) + (partial[0] if partial is not None else 0.0))
        hf, _ = orc.attnres_route([emb] + summaries + [mid[None]], f64(w_ffn))
        xf = f64(vw["x_hat"])[0]
        assert orc.max_rel_err(xf, orc.rmsnorm(hf)[0]) <= BF16_TOL, l
        u = f64(vw["ffn"])[0]
        assert orc.max_rel_err(u, orc.silu(mx(xf, wo[l]["up"]))) <= BF16_TOL, l
        nsum = len(summaries)
        new = f64(vw["blocks"][nsum])
        assert orc.max_rel_err(new[0], mid + mx(u, wo[l]["down"])) <= BF16_TOL, l
        partial = new
        if (l + 1) % span == 0:
            summaries.append(partial)
            partial = None
