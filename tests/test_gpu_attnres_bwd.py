"""GPU parity of the AttnRes route backward (sana_attnres_route_bwd) against
the float64 oracle's chain-rule gradients (pinned by finite differences).

Bars: source gradients (bf16 outputs) max relative error <= 2e-2; dw (fp32,
summed over all tokens) <= 1e-3."""

import numpy as np
import pytest
import torch

import sana_inputs as si
from oracle import sana_oracle as orc
from tests._sana import sana

pytestmark = pytest.mark.gpu


def f64(t):
    return si.as_f64(t)


@pytest.mark.parametrize("S,B,N,C", [(1, 1, 37, 256), (2, 2, 37, 512), (3, 2, 301, 768),
                                     (4, 1, 129, 256), (3, 1, 64, 4096)])
def test_small_matches_the_oracle(S, B, N, C):
    srcs = si.attnres_sources(7, S, B, N, C)
    w, _ = si.router_queries(7, C)
    dh = si.normal(9800 + S, (B, N, C))
    grads, dw = sana.attnres_route_bwd([t.cuda() for t in srcs], w.cuda(), dh.cuda())
    sana.sync_status()
    ref, dw_ref = orc.attnres_route_backward([f64(t) for t in srcs], f64(w), f64(dh))
    for i in range(S):
        assert orc.max_rel_err(f64(grads[i].cpu()), ref[i]) <= 2e-2, i
    assert orc.max_rel_err(dw.cpu().double().numpy(), dw_ref) <= 1e-3


def test_deterministic_and_no_tokens():
    srcs = [t.cuda() for t in si.attnres_sources(8, 3, 1, 5000, 3072)]
    w, _ = (t.cuda() for t in si.router_queries(8, 3072))
    dh = si.normal(9810, (1, 5000, 3072)).cuda()
    a = sana.attnres_route_bwd(srcs, w, dh)
    b = sana.attnres_route_bwd(srcs, w, dh)
    sana.sync_status()
    assert torch.equal(a[1], b[1]) and all(torch.equal(x, y) for x, y in zip(a[0], b[0]))
    e = [torch.empty(1, 0, 3072, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    g, dw = sana.attnres_route_bwd(e, w, e[0])
    sana.sync_status()
    assert bool((dw == 0).all())


def test_720p_three_sources():
    """The stack's case: 3 sources of the 720p/5s grid (N = 75,600, C = 3072);
    dw over all tokens (oracle in token chunks), source gradients on samples."""
    N, C = si.P720.N, si.P720.C
    srcs = si.attnres_sources(5, 3, 1, N, C)
    w, _ = si.router_queries(5, C)
    dh = si.normal(9820, (1, N, C))
    grads, dw = sana.attnres_route_bwd([t.cuda() for t in srcs], w.cuda(), dh.cuda())
    sana.sync_status()
    grads = [g.cpu() for g in grads]
    dw_ref = np.zeros(C)
    rows = set(np.random.default_rng(13).choice(N, size=512, replace=False).tolist())
    worst = 0.0
    for n0 in range(0, N, 4096):
        sl = slice(n0, min(N, n0 + 4096))
        ref, dwc = orc.attnres_route_backward([f64(t[:, sl]) for t in srcs], f64(w), f64(dh[:, sl]))
        dw_ref += dwc
        pick = np.array(sorted(r - n0 for r in rows if n0 <= r < sl.stop))
        if len(pick):
            for i in range(3):
                worst = max(worst, orc.max_rel_err(f64(grads[i][:, sl][:, pick]), ref[i][:, pick]))
    assert worst <= 2e-2
    assert orc.max_rel_err(dw.cpu().double().numpy(), dw_ref) <= 1e-3
