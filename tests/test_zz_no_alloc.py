"""The allocation-free linear-attention entry point.

sana_linattn_fwd_noalloc serves callers that cannot allocate device memory
(their device memory is owned by a framework they do not control, or they may
only use the buffers they are handed): it takes its scratch space from a fixed
array inside the library.  These tests call it through the C ABI twice in a
row and check each result against sana_linattn_fwd with a caller-provided
workspace.  Both run the same deterministic kernels with a fixed-order
combine, so the results must be bit-identical: any stale or overlapping use
of the shared array would show as a difference.  The file sits on its own so
that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import sana_inputs as si
from oracle import sana_oracle as orc
from tests._sana import _lib, sana

pytestmark = pytest.mark.gpu

F32_TOL = 1e-4


def _fn():
    f = _lib.lib.sana_linattn_fwd_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(_lib.Shape), ctypes.c_int] + [ctypes.c_void_p] * 4 + \
        [ctypes.POINTER(_lib.RopeStruct), ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    return f


def _call(q, k, v, g, rope, grid, heads, D):
    B = q.shape[0]
    shape = _lib.make_shape(B, grid, heads, D)
    out = torch.full_like(q, float("nan"))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = _fn()(ctypes.byref(shape), _lib._dtype_code(q), q.data_ptr(), k.data_ptr(), v.data_ptr(),
               None if g is None else g.data_ptr(), ctypes.byref(rope.struct), 1e-6,
               out.data_ptr(), stream)
    assert st == _lib.SANA_OK, _lib.last_error()
    sana.sync_status()
    return out


@pytest.mark.parametrize("B,heads,grid,gate", [(1, 2, (3, 5, 9), True), (1, 24, (21, 45, 80), True),
                                               (2, 4, (2, 8, 8), False), (1, 127, (1, 2, 64), True)])
def test_noalloc_matches_workspace_entry_point(B, heads, grid, gate):
    """Bit-identical to sana_linattn_fwd on two calls in a row; 127 (batch,
    head) pairs is the largest count whose scratch fits the array at D = 128."""
    N = grid[0] * grid[1] * grid[2]
    C = heads * 128
    q, k, v, g = (si.normal(14000 + 10 * N + i, (B, N, C)).cuda() for i in range(4))
    if not gate:
        g = None
    rope = sana.Rope(grid[0], grid[1], grid[2], (22, 21, 21))
    ref = sana.linattn_fwd(q, k, v, g, rope, grid, heads)
    sana.sync_status()
    for _ in range(2):
        out = _call(q, k, v, g, rope, grid, heads, 128)
        assert torch.equal(out, ref)


def test_noalloc_fp32_after_a_larger_call():
    """An fp32 call of a tiny shape, made right after a large bf16 call has
    filled the array, against the float64 oracle and against the workspace
    entry point."""
    grid, heads = (21, 45, 80), 24
    big = [si.normal(14500 + i, (1, 75600, 3072)).cuda() for i in range(3)]
    _call(big[0], big[1], big[2], None, sana.Rope(*grid, (22, 21, 21)), grid, heads, 128)
    del big
    wl = si.TINY
    tg = (wl.T, wl.H, wl.W)
    q, k, v, g = (si.normal(14600 + i, (wl.B, wl.N, wl.C), torch.float32) for i in range(4))
    rope = sana.Rope(*tg, wl.rope_split)
    ref = sana.linattn_fwd(q.cuda(), k.cuda(), v.cuda(), g.cuda(), rope, tg, wl.heads)
    sana.sync_status()
    yo, _, _ = orc.linattn_bidirectional(si.as_f64(q), si.as_f64(k), si.as_f64(v), tg,
                                         wl.rope_split, wl.heads, gate=si.as_f64(g))
    for _ in range(2):
        out = _call(q.cuda(), k.cuda(), v.cuda(), g.cuda(), rope, tg, wl.heads, wl.D)
        assert torch.equal(out, ref)
        assert orc.max_rel_err(si.as_f64(out), yo) <= F32_TOL
        assert np.isfinite(si.as_f64(out)).all()


@pytest.mark.parametrize("B,heads", [(1, 128), (4, 64)])
def test_noalloc_rejects_shapes_beyond_its_scratch(B, heads):
    """128 or more (batch, head) pairs need more than the 16 MiB array at
    D = 128 (bf16); the call is refused before anything is launched."""
    shape = _lib.make_shape(B, (1, 8, 8), heads, 128)
    rope = sana.Rope(1, 8, 8, (22, 21, 21))
    st = _fn()(ctypes.byref(shape), _lib.SANA_BF16, 256, 512, 768, None, ctypes.byref(rope.struct),
               1e-6, 1024, None)
    assert st == _lib.SANA_ERR_UNSUPPORTED and "scratch" in _lib.last_error()
    cap = _lib.lib.sana_linattn_noalloc_scratch_bytes
    cap.restype = ctypes.c_size_t
    assert sana.linattn_workspace_size(B, (1, 8, 8), heads, 128, _lib.SANA_BF16) > cap()
