"""The allocation-free linear-attention entry point.

sana_linattn_fwd_noalloc serves callers that cannot allocate device memory
(their device memory is owned by a framework they do not control, or they may
only use the buffers they are handed): it takes its scratch space from a fixed
array inside the library.  This test calls it through the C ABI twice in a row
and checks each result against sana_linattn_fwd with a caller-provided
workspace, within the bf16 tolerance the other tests use.  It sits in a file
of its own so that pytest collects it last.
"""

import ctypes

import pytest
import torch

import sana_inputs as si
from oracle import sana_oracle as orc
from tests._sana import _lib, sana

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


def _fn():
    f = _lib.lib.sana_linattn_fwd_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(_lib.Shape), ctypes.c_int] + [ctypes.c_void_p] * 4 + \
        [ctypes.POINTER(_lib.RopeStruct), ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    return f


@pytest.mark.parametrize("B,heads,grid,gate", [(1, 2, (3, 5, 9), True), (1, 24, (21, 45, 80), True),
                                               (2, 4, (2, 8, 8), False)])
def test_noalloc_matches_workspace_entry_point(B, heads, grid, gate):
    N = grid[0] * grid[1] * grid[2]
    C = heads * 128
    q, k, v, g = (si.normal(14000 + 10 * N + i, (B, N, C)).cuda() for i in range(4))
    if not gate:
        g = None
    rope = sana.Rope(grid[0], grid[1], grid[2], (22, 21, 21))
    ref = sana.linattn_fwd(q, k, v, g, rope, grid, heads)
    shape = _lib.make_shape(B, grid, heads, 128)
    f = _fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        st = f(ctypes.byref(shape), _lib.SANA_BF16, q.data_ptr(), k.data_ptr(), v.data_ptr(),
               None if g is None else g.data_ptr(), ctypes.byref(rope.struct), 1e-6,
               out.data_ptr(), stream)
        assert st == _lib.SANA_OK, _lib.last_error()
        sana.sync_status()
        assert orc.max_rel_err(si.as_f64(out), si.as_f64(ref)) <= BF16_TOL


def test_noalloc_rejects_shapes_beyond_its_scratch():
    shape = _lib.make_shape(4, (1, 8, 8), 64, 128)   # 256 (batch, head) states
    rope = sana.Rope(1, 8, 8, (22, 21, 21))
    st = _fn()(ctypes.byref(shape), _lib.SANA_BF16, 256, 512, 768, None, ctypes.byref(rope.struct),
               1e-6, 1024, None)
    assert st == _lib.SANA_ERR_UNSUPPORTED and "scratch" in _lib.last_error()
