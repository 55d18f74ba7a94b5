"""GPU parity of the MX block-scaled projection (MXFP8 activations, MXFP4
weights) against the float64 oracle ("SANA-Video 2.0" hyper.ai summary,
Experiments: only the linear GEMMs are quantised).

The quantisers are integer work and must match the oracle's codes and block
exponents exactly (the element codes are decoded from their bit fields here,
independently of both sides).  The GEMM multiplies exactly representable
products and accumulates in fp32; its bf16 output is held to the bf16 bar
against the oracle's float64 product of the dequantised operands."""

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


def _decode_e4m3(codes):
    c = codes.astype(np.int64)
    sign, e, m = c >> 7, (c >> 3) & 15, c & 7
    mag = np.where(e == 0, m / 8 * 2.0 ** -6, (1 + m / 8) * 2.0 ** (e - 7))
    assert not np.any((e == 15) & (m == 7)), "NaN code"
    return np.where(sign == 1, -mag, mag)


def _decode_e2m1(packed):
    p = packed.astype(np.int64)
    nib = np.stack([p & 15, p >> 4], axis=-1).reshape(*p.shape[:-1], -1)  # low nibble first
    sign, e, m = nib >> 3, (nib >> 1) & 3, nib & 1
    mag = np.where(e == 0, m * 0.5, (1 + m / 2) * 2.0 ** (e - 1))
    return np.where(sign == 1, -mag, mag)


def _scales(sf, rows, K):
    """Block exponents s = byte - 127 read from the documented atom layout."""
    b = sf.cpu().numpy().astype(np.int64)
    r = np.arange(rows)[:, None]
    blk = np.arange(K // 32)[None, :]
    atom = (r // 128) * (K // 128) + blk // 4
    off = atom * 512 + 16 * (r % 32) + 4 * ((r // 32) % 4) + blk % 4
    return b[off] - 127


def _special_rows(x):
    """Blocks the scale rule treats specially: all zero, huge, tiny, one spike."""
    x = x.clone()
    x[0, :32] = 0
    x[1, 32:64] *= 2.0 ** 60
    x[2, :32] *= 2.0 ** -100
    x[3, 64:96] = 0
    x[3, 70] = -3.0e4
    x[4, :] = torch.linspace(-7, 7, x.shape[1])
    return x


@pytest.mark.parametrize("rows,K", [(300, 256), (1, 128), (129, 384)])
@pytest.mark.parametrize("fp4", [False, True])
def test_quantiser_matches_the_oracle_bit_for_bit(rows, K, fp4):
    x = _special_rows(si.normal(16000 + rows + K, (max(rows, 8), K)))[:rows].contiguous()
    q, sf = sana.mx_quantize(x.cuda(), fp4=fp4)
    sana.sync_status()
    fmt = orc.E2M1 if fp4 else orc.E4M3
    el, s = orc.mx_quantize(f64(x), fmt)
    got = _decode_e2m1(q.cpu().numpy()) if fp4 else _decode_e4m3(q.cpu().numpy())
    np.testing.assert_array_equal(_scales(sf, rows, K), s)
    np.testing.assert_array_equal(got, el)
    # padding rows of the last atom hold scale 0
    if rows % 128:
        pad = np.arange(rows, (rows + 127) // 128 * 128)
        full = np.arange(K // 32)
        atom = (pad[:, None] // 128) * (K // 128) + full[None, :] // 4
        off = atom * 512 + 16 * (pad[:, None] % 32) + 4 * ((pad[:, None] // 32) % 4) + full % 4
        assert np.all(sf.cpu().numpy()[off] == 0)


@pytest.mark.parametrize("M,N,K", [(300, 256, 256), (1, 128, 128), (1000, 384, 1024),
                                   (77, 1280, 512)])
def test_gemm_matches_the_oracle(M, N, K):
    x = si.normal(16100 + M, (M, K))
    w = si.normal(16200 + N, (N, K), scale=K ** -0.5)
    xq, xs = sana.mx_quantize(x.cuda())
    wq, wsc = sana.mx_quantize(w.cuda(), fp4=True)
    y = sana.mx_gemm(xq, xs, wq, wsc, N)
    y2 = sana.mx_linear(x.cuda(), wq, wsc, N)
    sana.sync_status()
    ref = orc.mx_linear(f64(x), f64(w))
    err = orc.max_rel_err(f64(y), ref)
    print(f"mx gemm {M}x{N}x{K}: max_rel {err:.3e} elementwise "
          f"{orc.elementwise_rel_err(f64(y), ref):.3e}")
    assert err <= BF16_TOL, err
    assert torch.equal(y, y2)


def test_gemm_epilogues():
    M, N, K = 200, 256, 256
    x = si.normal(16300, (M, K))
    w = si.normal(16301, (N, K), scale=K ** -0.5)
    xq, xs = sana.mx_quantize(x.cuda())
    wq, wsc = sana.mx_quantize(w.cuda(), fp4=True)
    ref = orc.mx_linear(f64(x), f64(w))
    y = sana.mx_gemm(xq, xs, wq, wsc, N, epilogue=sana.EPI_SILU)
    sana.sync_status()
    assert orc.max_rel_err(f64(y), orc.silu(ref)) <= BF16_TOL
    base = si.normal(16302, (M, N))
    y = base.cuda().clone()
    sana.mx_gemm(xq, xs, wq, wsc, N, out=y, epilogue=sana.EPI_RESIDUAL)
    sana.sync_status()
    assert orc.max_rel_err(f64(y), f64(base) + ref) <= BF16_TOL


def test_quantised_error_is_the_formats_not_the_kernels():
    """Against the unquantised float64 product the MX projection is off by
    the formats' rounding (E2M1 has one mantissa bit), far more than the bf16
    bar; against the oracle of the quantised operands it is within it."""
    M, N, K = 256, 256, 512
    x = si.normal(16400, (M, K))
    w = si.normal(16401, (N, K), scale=K ** -0.5)
    wq, wsc = sana.mx_quantize(w.cuda(), fp4=True)
    y = sana.mx_linear(x.cuda(), wq, wsc, N)
    sana.sync_status()
    exact = f64(x) @ f64(w).T
    assert orc.max_rel_err(f64(y), exact) > 4 * orc.max_rel_err(f64(y), orc.mx_linear(f64(x), f64(w)))


def test_720p_qkvg_projection_sampled_rows():
    """The stack's QKVG projection at 720p/5s: (75,600 x 3072) . (12,288 x 3072)^T,
    checked on sampled rows and the ragged last row tile."""
    M, C = si.P720.N, si.P720.C
    x = si.normal(16500, (M, C))
    w = si.normal(16501, (4 * C, C), scale=C ** -0.5)
    wq, wsc = sana.mx_quantize(w.cuda(), fp4=True)
    y = sana.mx_linear(x.cuda(), wq, wsc, 4 * C)
    sana.sync_status()
    rows = np.unique(np.concatenate([np.random.default_rng(8).choice(M, 256, replace=False),
                                     np.arange(M - 80, M)]))
    ref = orc.mx_linear(f64(x[rows]), f64(w))
    err = orc.max_rel_err(f64(y[rows]), ref)
    print(f"mx qkvg 720p sampled rows: max_rel {err:.3e}")
    assert err <= BF16_TOL, err
