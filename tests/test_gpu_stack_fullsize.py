"""Full-size parity of the hybrid stack at the 720p/5s shape (N = 75,600,
24 heads x 128, hidden 3072), teacher-forced step by step.

The float64 oracle cannot run a whole 720p stack (its projections alone are
tens of TFLOP per layer), so each step of each layer is checked on its own:
the stack is run for the first l + 1 layers, its intermediates are read from
the workspace (sana_hybrid_stack_workspace_layout), and every step's GPU
output is compared with the oracle's step applied to the GPU's own input of
that step:

* AttnRes route + RMSNorm + QKVG projection, on sampled rows;
* the attention (linear layers: the oracle's state from the GPU's full K and
  V, then the sampled query rows; anchors: the sampled query rows against
  all 75,600 keys);
* the W_o projection into the partial sum (or the residual stream);
* the FFN route + RMSNorm, the SiLU up-projection and the down-projection
  into the partial sum;
* the stack's output (the final route over the sources).

Sampled rows: 256 seeded rows, the first 8 tokens and the last 80 (the
ragged last 128-token tile).  Each comparison uses the parity bar (max
relative error 2e-2 for bf16); the elementwise measure is printed beside it.

Pages: "SANA-Video 2.0" abstract (three gated linear layers to one gated
softmax anchor); hyper.ai summary, Method (the AttnRes equation, the shared
router queries, block summaries every 8 layers).
"""

import numpy as np
import pytest
import torch

import sana_inputs as si
from oracle import sana_oracle as orc
from tests._sana import sana

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

BF16_TOL = 2e-2
WL = si.STACK
GRID = (WL.T, WL.H, WL.W)
SPLIT = WL.rope_split
N, C, HEADS, D = WL.N, WL.C, WL.heads, WL.D


def f64(t):
    return si.as_f64(t)


def _rows():
    rng = np.random.default_rng(2024)
    r = np.concatenate([rng.choice(N, 256, replace=False), np.arange(8), np.arange(N - 80, N)])
    return np.unique(r)


ROWS = _rows()
ROWS_T = torch.from_numpy(ROWS)
ANG = orc.rope_angles(*GRID, *SPLIT)


def _check(name, got, ref, log):
    err = orc.max_rel_err(got, ref)
    ew = orc.elementwise_rel_err(got, ref)
    log.append((name, err, ew))
    print(f"{name:38s} max_rel {err:.3e}  elementwise {ew:.3e}")
    assert err <= BF16_TOL, (name, err)


def _oracle_attention_rows(q, k, v, g, anchor):
    """The gated attention of the GPU's own Q, K, V, G (CPU bf16, (1, N, C))
    at the sampled query rows, head by head."""
    out = np.empty((1, len(ROWS), C))
    for h in range(HEADS):
        sl = slice(h * D, (h + 1) * D)
        kh, vh = f64(k[..., sl]), f64(v[..., sl])
        if anchor:
            out[..., sl] = orc.softmax_anchor(f64(q[..., sl]), kh, vh, GRID, SPLIT, 1,
                                              gate=f64(g[..., sl]), rows=ROWS)
        else:
            S, z = orc.linattn_state(kh, vh, ANG, 1)
            out[..., sl] = orc.linattn_apply(f64(q[:, ROWS_T, sl]), S, z, ANG[ROWS], 1,
                                             gate=f64(g[:, ROWS_T, sl]))
    return out


class _Stack:
    """The stack's inputs on the device and a workspace sized for all layers."""

    def __init__(self, config, layers, use_attnres, ffn_mult):
        self.layers, self.use_attnres, self.ffn_mult = layers, use_attnres, ffn_mult
        self.x = si.normal(si.seed_of(config, si.G_ID), (1, N, C))
        self.w = si.projection_weights(config, layers, C, ffn_mult)
        self.w_attn, self.w_ffn = si.router_queries(config, C)
        self.wd = [{k: t.cuda() for k, t in d.items()} for d in self.w]
        self.xd = self.x.cuda()
        self.rope = sana.Rope(*GRID, SPLIT)
        self.ws = torch.empty(sana.hybrid_stack_workspace_size(1, GRID, HEADS, self.cfg(layers)),
                              dtype=torch.uint8, device="cuda")

    def cfg(self, layers):
        return sana.stack_config(layers, block_span=8, use_attnres=self.use_attnres,
                                 ffn_mult=self.ffn_mult)

    def run(self, layers):
        cfg = self.cfg(layers)
        out = sana.hybrid_stack_fwd(self.xd, self.wd[:layers], self.w_attn.cuda(),
                                    self.w_ffn.cuda(), self.rope, GRID, HEADS, cfg, ws=self.ws)
        sana.sync_status()
        return sana.hybrid_stack_workspace_views(self.ws, 1, GRID, HEADS, cfg), out

    def weight(self, l, key):
        return f64(self.w[l][key])


def _rows_of(t):
    return f64(t[:, ROWS_T.to(t.device)])


def test_group_720p_teacher_forced():
    """Three gated linear layers then one gated softmax anchor, plain pre-norm
    residual, no FFN (the 720p/5s hybrid group)."""
    st = _Stack(3, 4, False, 0)
    log = []
    prev = _rows_of(st.x)            # residual stream before layer l, sampled rows
    for l in range(4):
        views, out = st.run(l + 1)
        anchor = orc.is_anchor_layer(l)
        xhat = _rows_of(views["x_hat"])
        _check(f"L{l} rmsnorm", xhat, orc.rmsnorm(prev), log)
        qkvg = xhat @ st.weight(l, "qkvg").T
        for i, key in enumerate("qkvg"):
            _check(f"L{l} proj {key}", _rows_of(views[key]), qkvg[..., i * C:(i + 1) * C], log)
        q, k, v, g = (views[key].cpu() for key in "qkvg")
        attn = _rows_of(views["attn"])
        _check(f"L{l} {'anchor' if anchor else 'linear'} attention", attn,
               _oracle_attention_rows(q, k, v, g, anchor), log)
        new = _rows_of(out)
        _check(f"L{l} W_o residual", new, prev + attn @ st.weight(l, "o").T, log)
        prev = new
    assert len(log) == 4 * 7


def test_attnres_stack_720p_teacher_forced():
    """16 layers in two AttnRes blocks of 8, FFN 3C, 3:1 linear:anchor, shared
    router queries (the full-depth configuration)."""
    layers = 16
    st = _Stack(5, layers, True, 3)
    w_attn, w_ffn = f64(st.w_attn), f64(st.w_ffn)
    log = []
    emb = _rows_of(st.x)
    summaries, partial = [], None    # sampled rows of the sources before layer l
    for l in range(layers):
        views, out = st.run(l + 1)
        anchor = orc.is_anchor_layer(l)
        # attention sublayer: route -> RMSNorm -> QKVG
        srcs = [emb] + summaries + ([partial] if partial is not None else [])
        h, _ = orc.attnres_route(srcs, w_attn)
        qkvg = orc.rmsnorm(h) @ st.weight(l, "qkvg").T
        for i, key in enumerate("qkvg"):
            _check(f"L{l} route+proj {key}", _rows_of(views[key]), qkvg[..., i * C:(i + 1) * C], log)
        q, k, v, g = (views[key].cpu() for key in "qkvg")
        attn = _rows_of(views["attn"])
        _check(f"L{l} {'anchor' if anchor else 'linear'} attention", attn,
               _oracle_attention_rows(q, k, v, g, anchor), log)
        mid = attn @ st.weight(l, "o").T + (partial if partial is not None else 0.0)
        # FFN sublayer: route over the sources with the updated partial sum
        h, _ = orc.attnres_route([emb] + summaries + [mid], w_ffn)
        xhat = _rows_of(views["x_hat"])
        _check(f"L{l} ffn route+rmsnorm", xhat, orc.rmsnorm(h), log)
        u = _rows_of(views["ffn"])
        _check(f"L{l} ffn up+silu", u, orc.silu(xhat @ st.weight(l, "up").T), log)
        new = mid + u @ st.weight(l, "down").T
        nsum = len(summaries)
        _check(f"L{l} partial sum", _rows_of(views["blocks"][nsum]), new, log)
        partial = _rows_of(views["blocks"][nsum])
        if (l + 1) % 8 == 0:
            summaries.append(partial)
            partial = None
        # the stack's output after l + 1 layers: route over the final sources
        srcs = [emb] + summaries + ([partial] if partial is not None else [])
        h, _ = orc.attnres_route(srcs, w_attn)
        _check(f"L{l} output route", _rows_of(out), h, log)
    assert len(log) == layers * 9
