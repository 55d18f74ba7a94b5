"""C-ABI checks that need no GPU: the library loads, exports every symbol
include/sana.h declares, computes the RoPE tables on the host like the oracle,
and rejects bad arguments before touching the device."""

import ctypes
import os
import re

import numpy as np
import pytest

from tests._sana import _lib, sana
from oracle import sana_oracle as orc

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "sana.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sana_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 15
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_error_string():
    assert b"sm_100a" in _lib.lib.sana_version()
    assert isinstance(_lib.last_error(), str)


@pytest.mark.parametrize("grid,split,t_total", [((2, 4, 4), (2, 3, 3), 2), ((21, 45, 80), (22, 21, 21), 21),
                                                ((3, 45, 80), (22, 21, 21), 241)])
def test_host_rope_tables_match_oracle_angles(grid, split, t_total):
    T, H, W = grid
    tab = _lib.host_rope_tables(t_total, H, W, split).numpy().astype(np.float64)
    n_t, n_h, n_w = split
    off = 0
    parts = {}
    for name, npos, npair in (("t", t_total, n_t), ("h", H, n_h), ("w", W, n_w)):
        c = tab[off:off + npos * npair].reshape(npos, npair)
        s = tab[off + npos * npair:off + 2 * npos * npair].reshape(npos, npair)
        parts[name] = (c, s)
        off += 2 * npos * npair
    # oracle angles for the frames [t0, t0 + T)
    t0 = t_total - T
    ang = orc.rope_angles(T, H, W, *split, t_offset=t0)
    t, h, w = orc.token_grid(T, H, W, t0)
    got_c = np.concatenate([parts["t"][0][t], parts["h"][0][h], parts["w"][0][w]], axis=1)
    got_s = np.concatenate([parts["t"][1][t], parts["h"][1][h], parts["w"][1][w]], axis=1)
    # fp32 rounding of cos / sin evaluated in double
    assert np.max(np.abs(got_c - np.cos(ang))) < 1e-7
    assert np.max(np.abs(got_s - np.sin(ang))) < 1e-7


def _shape(**kw):
    d = dict(B=1, T=2, H=4, W=4, heads=2, head_dim=16, t_offset=0)
    d.update(kw)
    return _lib.Shape(d["B"], d["T"], d["H"], d["W"], d["heads"], d["head_dim"], d["t_offset"])


def test_workspace_sizes():
    L = _lib.lib
    assert L.sana_linattn_workspace_size(ctypes.byref(_shape()), _lib.SANA_F32) > 0
    s720 = _shape(T=21, H=45, W=80, heads=24, head_dim=128)
    ws = L.sana_linattn_workspace_size(ctypes.byref(s720), _lib.SANA_BF16)
    # 6 splits x 24 heads of (128x128 + 128) fp32 partials, S^T in bf16, z: about 10 MB
    assert 9e6 < ws < 12e6
    assert L.sana_softmax_anchor_workspace_size(ctypes.byref(s720), _lib.SANA_BF16) >= 2 * 75600 * 3072 * 2
    # unsupported shapes report 0
    assert L.sana_linattn_workspace_size(ctypes.byref(_shape(head_dim=64)), _lib.SANA_BF16) == 0


def _call_fwd(shape, dtype, ptr=16, rope=None, eps=1e-6, ws_bytes=1 << 20):
    r = rope or _lib.RopeStruct(16, 16, 16, 16, 16, 16, 2, 3, 3, 2, 4, 4)
    return _lib.lib.sana_linattn_fwd(ctypes.byref(shape) if shape is not None else None, dtype,
                                     ptr, ptr + 4096, ptr + 8192, None, ctypes.byref(r), eps,
                                     ptr + 16384, 1 << 20, ws_bytes, None)


def test_validation_errors_return_before_any_device_work():
    L = _lib
    # NULL shape
    assert _call_fwd(None, L.SANA_F32) == L.SANA_ERR_INVALID_ARG
    # bf16 requires head_dim 128
    assert _call_fwd(_shape(head_dim=16), L.SANA_BF16) == L.SANA_ERR_UNSUPPORTED
    assert "head_dim" in L.last_error()
    # fp32 head_dim outside {16, 32, 64, 128}
    assert _call_fwd(_shape(head_dim=24), L.SANA_F32) == L.SANA_ERR_UNSUPPORTED
    # rope split not covering head_dim / 2
    bad = _lib.RopeStruct(16, 16, 16, 16, 16, 16, 2, 3, 2, 2, 4, 4)
    assert _call_fwd(_shape(), L.SANA_F32, rope=bad) == L.SANA_ERR_INVALID_ARG
    # tables that do not cover the frames
    short = _lib.RopeStruct(16, 16, 16, 16, 16, 16, 2, 3, 3, 1, 4, 4)
    assert _call_fwd(_shape(), L.SANA_F32, rope=short) == L.SANA_ERR_INVALID_ARG
    # misaligned pointer
    assert _call_fwd(_shape(), L.SANA_F32, ptr=18) == L.SANA_ERR_INVALID_ARG
    # negative eps
    assert _call_fwd(_shape(), L.SANA_F32, eps=-1.0) == L.SANA_ERR_INVALID_ARG
    # workspace too small
    assert _call_fwd(_shape(), L.SANA_F32, ws_bytes=16) == L.SANA_ERR_WORKSPACE
    # output aliasing an input
    r = _lib.RopeStruct(16, 16, 16, 16, 16, 16, 2, 3, 3, 2, 4, 4)
    st = L.lib.sana_linattn_fwd(ctypes.byref(_shape()), L.SANA_F32, 4096, 8192, 12288, None,
                                ctypes.byref(r), 1e-6, 4096, 1 << 20, 1 << 20, None)
    assert st == L.SANA_ERR_INVALID_ARG and "alias" in L.last_error()


def _call_scan(shape, frames, S=8 << 20, z=9 << 20, ws_bytes=1 << 24, out=4 << 20):
    # fake device addresses, 1 MiB apart: every call here fails validation first
    r = _lib.RopeStruct(16, 16, 16, 16, 16, 16, 2, 3, 3, 8, 4, 4)
    return _lib.lib.sana_linattn_block_causal_scan(
        ctypes.byref(shape), frames, _lib.SANA_F32, 1 << 20, 2 << 20, 3 << 20, None,
        ctypes.byref(r), 1e-6, S, z, 1, out, 1 << 26, ws_bytes, None)


def test_block_causal_scan_sizes_and_validation():
    L = _lib
    # 720p/60s: 80 blocks of 3 frames (one split each: 80 x 24 CTAs fill the
    # GPU) + a 1-frame block (148 // 24 = 6 splits), then 81 prefix states
    long_seq = _shape(T=241, H=45, W=80, heads=24, head_dim=128)
    ws = L.lib.sana_linattn_block_causal_scan_workspace_size(ctypes.byref(long_seq), 3, L.SANA_BF16)
    per_state = 24 * (128 * 128 + 128) * 4
    want = (80 + 6 + 81) * per_state
    assert want <= ws < want + 8 * 256
    assert L.lib.sana_linattn_block_causal_scan_workspace_size(ctypes.byref(long_seq), 0,
                                                               L.SANA_BF16) == 0
    s = _shape(T=8)
    assert _call_scan(s, 0) == L.SANA_ERR_INVALID_ARG and "chunk_frames" in L.last_error()
    assert _call_scan(s, 3, S=None) == L.SANA_ERR_INVALID_ARG
    assert _call_scan(s, 3, S=(8 << 20) + 4) == L.SANA_ERR_INVALID_ARG
    assert _call_scan(s, 3, ws_bytes=64) == L.SANA_ERR_WORKSPACE
    assert _call_scan(s, 3, out=2 << 20) == L.SANA_ERR_INVALID_ARG and "alias" in L.last_error()


def test_sparse_anchor_sizes_and_validation():
    L = _lib
    s720 = _shape(T=21, H=45, W=80, heads=24, head_dim=128)
    ws = L.lib.sana_softmax_anchor_sparse_workspace_size(ctypes.byref(s720), L.SANA_BF16)
    # rotated Q and K (2 x 464.5 MB) + per-tile fp32 sums of both (2 x 591 x 3072 x 4 B)
    assert ws >= 2 * 75600 * 3072 * 2 + 2 * 591 * 3072 * 4
    assert L.lib.sana_softmax_anchor_sparse_workspace_size(ctypes.byref(_shape()), L.SANA_F32) == 0
    r = _lib.RopeStruct(16, 16, 16, 16, 16, 16, 22, 21, 21, 2, 4, 4)
    s = _shape(head_dim=128)  # N = 32: one key tile

    def call(dtype=L.SANA_BF16, keep=1, tiles=6 << 20, ws_bytes=1 << 24):
        return L.lib.sana_softmax_anchor_sparse_fwd(
            ctypes.byref(s), dtype, 1 << 20, 2 << 20, 3 << 20, None, ctypes.byref(r), 0.0, keep,
            tiles, 1, 4 << 20, 1 << 26, ws_bytes, None)
    assert call(dtype=L.SANA_F32) == L.SANA_ERR_UNSUPPORTED
    assert call(keep=0) == L.SANA_ERR_INVALID_ARG and "keep_tiles" in L.last_error()
    assert call(keep=2) == L.SANA_ERR_INVALID_ARG
    assert call(tiles=None) == L.SANA_ERR_INVALID_ARG
    assert call(tiles=4 << 20) == L.SANA_ERR_INVALID_ARG and "alias" in L.last_error()
    assert call(ws_bytes=64) == L.SANA_ERR_WORKSPACE


def test_backward_validation():
    L = _lib
    s = _shape(head_dim=128)
    assert L.lib.sana_linattn_bwd_workspace_size(ctypes.byref(s), L.SANA_BF16) > 0
    assert L.lib.sana_linattn_bwd_workspace_size(ctypes.byref(_shape()), L.SANA_F32) == 0
    r = _lib.RopeStruct(16, 16, 16, 16, 16, 16, 22, 21, 21, 2, 4, 4)
    M = 1 << 20

    def call(dtype=L.SANA_BF16, g=None, dg=None, dq=5 * M, ws_bytes=1 << 26):
        return L.lib.sana_linattn_bwd(ctypes.byref(s), dtype, M, 2 * M, 3 * M, g, ctypes.byref(r),
                                      1e-6, 4 * M, dq, 6 * M, 7 * M, dg, 1 << 28, ws_bytes, None)
    assert call(dtype=L.SANA_F32) == L.SANA_ERR_UNSUPPORTED
    assert call(g=8 * M) == L.SANA_ERR_INVALID_ARG and "d_gate" in L.last_error()
    assert call(dq=2 * M) == L.SANA_ERR_INVALID_ARG and "alias" in L.last_error()
    assert call(ws_bytes=64) == L.SANA_ERR_WORKSPACE

    def saved(S=9 * M, z=10 * M, dq=5 * M, ws=1 << 28):
        return L.lib.sana_linattn_bwd_saved_state(
            ctypes.byref(s), L.SANA_BF16, M, 2 * M, 3 * M, None, ctypes.byref(r), 1e-6, S, z,
            4 * M, dq, 6 * M, 7 * M, None, ws, 1 << 26, None)
    assert saved(S=None) == L.SANA_ERR_INVALID_ARG and "saved state" in L.last_error()
    assert saved(z=None) == L.SANA_ERR_INVALID_ARG
    assert saved(S=9 * M + 4) == L.SANA_ERR_INVALID_ARG and "aligned" in L.last_error()
    assert saved(dq=9 * M) == L.SANA_ERR_INVALID_ARG and "saved state" in L.last_error()
    assert saved(ws=9 * M) == L.SANA_ERR_INVALID_ARG and "workspace" in L.last_error()
    assert saved(dq=2 * M) == L.SANA_ERR_INVALID_ARG and "alias" in L.last_error()


def test_attnres_and_gemm_validation():
    L = _lib
    arr = (ctypes.c_void_p * 1)(4096)
    assert L.lib.sana_attnres_route(1, 10, 64, L.SANA_BF16, arr, 0, 8192, 1e-6, 16384, None, None) \
        == L.SANA_ERR_UNSUPPORTED
    assert L.lib.sana_attnres_route(1, 10, 60, L.SANA_BF16, arr, 1, 8192, 1e-6, 1 << 20, None, None) \
        == L.SANA_ERR_UNSUPPORTED
    assert L.lib.sana_gemm_bf16(128, 128, 100, 4096, 100, 8192, 1 << 20, 128, 0, None) \
        == L.SANA_ERR_UNSUPPORTED


@pytest.mark.parametrize("layers,span,attnres,ffn", [(16, 8, True, 3), (4, 8, False, 0),
                                                      (5, 2, True, 0), (8, 8, True, 3)])
def test_stack_workspace_layout_is_disjoint_and_inside_the_workspace(layers, span, attnres, ffn):
    """The intermediates the stack exposes lie inside its workspace, do not
    overlap, and there is one AttnRes buffer per started block."""
    grid, heads = (21, 45, 80), 24
    cfg = sana.stack_config(layers, block_span=span, use_attnres=attnres, ffn_mult=ffn)
    s = _lib.make_shape(1, grid, heads, 128)
    lay = _lib.StackWsLayout()
    assert _lib.lib.sana_hybrid_stack_workspace_layout(ctypes.byref(s), ctypes.byref(cfg),
                                                       ctypes.byref(lay)) == _lib.SANA_OK
    total = _lib.lib.sana_hybrid_stack_workspace_size(ctypes.byref(s), ctypes.byref(cfg))
    tok_bytes = grid[0] * grid[1] * grid[2] * heads * 128 * 2
    spans = [(getattr(lay, k), tok_bytes) for k in ("x_hat", "q", "k", "v", "g", "attn")]
    if ffn:
        spans.append((lay.ffn, ffn * tok_bytes))
    else:
        assert lay.ffn == 2 ** 64 - 1
    nblocks = -(-layers // span) if attnres else 0
    assert lay.num_blocks == nblocks
    spans += [(lay.blocks[i], tok_bytes) for i in range(nblocks)]
    spans.sort()
    for (a, na), (b, _) in zip(spans, spans[1:]):
        assert a + na <= b
    assert spans[-1][0] + spans[-1][1] <= total
    assert all(off % 256 == 0 for off, _ in spans)


def test_stack_workspace_layout_rejects_bad_arguments():
    cfg = sana.stack_config(4, block_span=8, use_attnres=False, ffn_mult=0)
    s = _lib.make_shape(1, (2, 4, 8), 2, 128)
    assert _lib.lib.sana_hybrid_stack_workspace_layout(ctypes.byref(s), ctypes.byref(cfg),
                                                       None) == _lib.SANA_ERR_INVALID_ARG
    bad = sana.stack_config(0, block_span=8)
    lay = _lib.StackWsLayout()
    assert _lib.lib.sana_hybrid_stack_workspace_layout(ctypes.byref(s), ctypes.byref(bad),
                                                       ctypes.byref(lay)) != _lib.SANA_OK


def test_mx_sizes_and_validation():
    """The MX projection's scale-atom sizes and argument checks (no device
    work: every call below fails validation first)."""
    L = _lib
    # 75,600 rows x 3072: 591 row atoms x 24 K atoms x 512 bytes
    assert L.lib.sana_mx_scale_bytes(75600, 3072) == 591 * 24 * 512
    assert L.lib.sana_mx_scale_bytes(1, 128) == 512
    assert L.lib.sana_mx_scale_bytes(10, 100) == 0
    assert L.lib.sana_mx_linear_workspace_size(300, 256) >= 300 * 256 + 3 * 2 * 512
    M = 1 << 20
    assert L.lib.sana_mx_quantize(M, 10, 100, 0, 2 * M, 3 * M, None) == L.SANA_ERR_INVALID_ARG
    assert L.lib.sana_mx_quantize(M, 10, 128, 2, 2 * M, 3 * M, None) == L.SANA_ERR_INVALID_ARG
    assert L.lib.sana_mx_quantize(M + 8, 10, 128, 1, 2 * M, 3 * M, None) == L.SANA_ERR_INVALID_ARG
    assert L.lib.sana_mx_quantize(M, 10, 128, 0, M, 3 * M, None) == L.SANA_ERR_INVALID_ARG
    g = L.lib.sana_mx_gemm
    assert g(256, 100, 256, M, 2 * M, 3 * M, 4 * M, 5 * M, 100, 0, None) == L.SANA_ERR_UNSUPPORTED
    assert g(256, 128, 192, M, 2 * M, 3 * M, 4 * M, 5 * M, 128, 0, None) == L.SANA_ERR_UNSUPPORTED
    assert g(256, 128, 256, M, 2 * M, 3 * M + 16, 4 * M, 5 * M, 128, 0, None) == \
        L.SANA_ERR_INVALID_ARG and "32-byte" in L.last_error()
    assert g(256, 128, 256, M, 2 * M, 3 * M, 4 * M, M, 128, 0, None) == L.SANA_ERR_INVALID_ARG
    assert g(256, 128, 256, M, 2 * M, 3 * M, 4 * M, 5 * M, 128, 3, None) == L.SANA_ERR_INVALID_ARG
    lin = L.lib.sana_mx_linear
    assert lin(300, 256, 256, M, 2 * M, 3 * M, 4 * M, 256, 0, 5 * M, 64, None) == L.SANA_ERR_WORKSPACE
