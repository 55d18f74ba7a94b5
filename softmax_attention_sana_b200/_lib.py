"""ctypes binding of libsana (include/sana.h).

Argument marshalling only: every step of the attention path runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  If libsana.so is missing the import fails loudly; there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, Structure, c_char_p, c_double, c_float, c_int, c_longlong, c_size_t,
                    c_void_p)

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsana.so")

SANA_OK, SANA_ERR_INVALID_ARG, SANA_ERR_UNSUPPORTED, SANA_ERR_WORKSPACE, SANA_ERR_CUDA, \
    SANA_ERR_TIMEOUT = range(6)
SANA_F32, SANA_BF16 = 0, 1
EPI_NONE, EPI_SILU, EPI_RESIDUAL = 0, 1, 2
STATUS_NAMES = {0: "SANA_OK", 1: "SANA_ERR_INVALID_ARG", 2: "SANA_ERR_UNSUPPORTED",
                3: "SANA_ERR_WORKSPACE", 4: "SANA_ERR_CUDA", 5: "SANA_ERR_TIMEOUT"}


class SanaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Shape(Structure):
    _fields_ = [("B", c_int), ("T", c_int), ("H", c_int), ("W", c_int), ("heads", c_int),
                ("head_dim", c_int), ("t_offset", c_int)]


class RopeStruct(Structure):
    _fields_ = [("cos_t", c_void_p), ("sin_t", c_void_p), ("cos_h", c_void_p), ("sin_h", c_void_p),
                ("cos_w", c_void_p), ("sin_w", c_void_p), ("n_t", c_int), ("n_h", c_int),
                ("n_w", c_int), ("T_total", c_int), ("H", c_int), ("W", c_int)]


class StackConfig(Structure):
    _fields_ = [("layers", c_int), ("block_span", c_int), ("ratio", c_int), ("use_attnres", c_int),
                ("ffn_mult", c_int), ("eps", c_float), ("rms_eps", c_float),
                ("anchor_scale", c_float), ("anchor_keep_tiles", c_int),
                ("mx_projections", c_int)]


class StackWeights(Structure):
    _fields_ = [("w_qkvg", POINTER(c_void_p)), ("w_o", POINTER(c_void_p)),
                ("w_up", POINTER(c_void_p)), ("w_down", POINTER(c_void_p)),
                ("w_attn", c_void_p), ("w_ffn", c_void_p),
                ("mx_qkvg", POINTER(c_void_p)), ("mx_qkvg_scales", POINTER(c_void_p)),
                ("mx_o", POINTER(c_void_p)), ("mx_o_scales", POINTER(c_void_p)),
                ("mx_up", POINTER(c_void_p)), ("mx_up_scales", POINTER(c_void_p)),
                ("mx_down", POINTER(c_void_p)), ("mx_down_scales", POINTER(c_void_p))]


class StackWsLayout(Structure):
    _fields_ = [("x_hat", c_size_t), ("q", c_size_t), ("k", c_size_t), ("v", c_size_t),
                ("g", c_size_t), ("attn", c_size_t), ("ffn", c_size_t), ("num_blocks", c_int),
                ("blocks", c_size_t * 16)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsana.so not built ({LIB_PATH}); run softmax_attention_sana_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "sana_version": (c_char_p, []),
        "sana_last_error_string": (c_char_p, []),
        "sana_rope_tables_count": (c_size_t, [c_int] * 6),
        "sana_rope_tables_host": (c_int, [c_int] * 6 + [c_double, c_void_p]),
        "sana_rope_bind": (c_int, [c_void_p] + [c_int] * 6 + [POINTER(RopeStruct)]),
        "sana_linattn_workspace_size": (c_size_t, [POINTER(Shape), c_int]),
        "sana_linattn_fwd": (c_int, [POINTER(Shape), c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                     POINTER(RopeStruct), c_float, c_void_p, c_void_p, c_size_t,
                                     c_void_p]),
        "sana_linattn_state_workspace_size": (c_size_t, [POINTER(Shape), c_int]),
        "sana_linattn_state": (c_int, [POINTER(Shape), c_int, c_void_p, c_void_p,
                                       POINTER(RopeStruct), c_void_p, c_void_p, c_void_p, c_size_t,
                                       c_void_p]),
        "sana_linattn_apply": (c_int, [POINTER(Shape), c_int, c_void_p, c_void_p,
                                       POINTER(RopeStruct), c_void_p, c_void_p, c_float, c_void_p,
                                       c_void_p]),
        "sana_linattn_block_causal_step": (c_int, [POINTER(Shape), c_int, c_void_p, c_void_p,
                                                   c_void_p, c_void_p, POINTER(RopeStruct), c_float,
                                                   c_void_p, c_void_p, c_int, c_void_p, c_void_p,
                                                   c_size_t, c_void_p]),
        "sana_linattn_block_causal_scan_workspace_size": (c_size_t, [POINTER(Shape), c_int, c_int]),
        "sana_linattn_block_causal_scan": (c_int, [POINTER(Shape), c_int, c_int, c_void_p, c_void_p,
                                                   c_void_p, c_void_p, POINTER(RopeStruct),
                                                   c_float, c_void_p, c_void_p, c_int, c_void_p,
                                                   c_void_p, c_size_t, c_void_p]),
        "sana_linattn_bwd_workspace_size": (c_size_t, [POINTER(Shape), c_int]),
        "sana_linattn_bwd": (c_int, [POINTER(Shape), c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                     POINTER(RopeStruct), c_float, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
        "sana_linattn_bwd_saved_state": (c_int, [POINTER(Shape), c_int, c_void_p, c_void_p,
                                                 c_void_p, c_void_p, POINTER(RopeStruct), c_float,
                                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                 c_void_p, c_void_p, c_void_p, c_size_t,
                                                 c_void_p]),
        "sana_softmax_anchor_workspace_size": (c_size_t, [POINTER(Shape), c_int]),
        "sana_softmax_anchor_fwd": (c_int, [POINTER(Shape), c_int, c_void_p, c_void_p, c_void_p,
                                            c_void_p, POINTER(RopeStruct), c_float, c_void_p,
                                            c_void_p, c_size_t, c_void_p]),
        "sana_rope_apply": (c_int, [POINTER(Shape), c_int, c_void_p, POINTER(RopeStruct), c_float,
                                    c_void_p, c_void_p]),
        "sana_softmax_anchor_rotated_fwd": (c_int, [POINTER(Shape), c_void_p, c_void_p, c_void_p,
                                                    c_void_p, c_void_p, c_void_p]),
        "sana_softmax_anchor_sparse_workspace_size": (c_size_t, [POINTER(Shape), c_int]),
        "sana_softmax_anchor_sparse_fwd": (c_int, [POINTER(Shape), c_int, c_void_p, c_void_p,
                                                   c_void_p, c_void_p, POINTER(RopeStruct),
                                                   c_float, c_int, c_void_p, c_int, c_void_p,
                                                   c_void_p, c_size_t, c_void_p]),
        "sana_attnres_route": (c_int, [c_int, c_longlong, c_int, c_int, POINTER(c_void_p), c_int,
                                       c_void_p, c_float, c_void_p, c_void_p, c_void_p]),
        "sana_attnres_route_bwd_workspace_size": (c_size_t, [c_int, c_longlong, c_int]),
        "sana_attnres_route_bwd": (c_int, [c_int, c_longlong, c_int, c_int, POINTER(c_void_p),
                                           c_int, c_void_p, c_float, c_void_p, POINTER(c_void_p),
                                           c_void_p, c_void_p, c_size_t, c_void_p]),
        "sana_gemm_bf16": (c_int, [c_longlong, c_int, c_int, c_void_p, c_longlong, c_void_p,
                                   c_void_p, c_longlong, c_int, c_void_p]),
        "sana_rmsnorm": (c_int, [c_longlong, c_int, c_int, c_void_p, c_float, c_void_p, c_void_p]),
        "sana_hybrid_stack_workspace_size": (c_size_t, [POINTER(Shape), POINTER(StackConfig)]),
        "sana_hybrid_stack_workspace_layout": (c_int, [POINTER(Shape), POINTER(StackConfig),
                                                       POINTER(StackWsLayout)]),
        "sana_hybrid_stack_fwd": (c_int, [POINTER(Shape), POINTER(StackConfig),
                                          POINTER(StackWeights), POINTER(RopeStruct), c_void_p,
                                          c_void_p, c_void_p, c_size_t, c_void_p]),
        "sana_mx_scale_bytes": (c_size_t, [c_longlong, c_int]),
        "sana_mx_quantize": (c_int, [c_void_p, c_longlong, c_int, c_int, c_void_p, c_void_p,
                                     c_void_p]),
        "sana_mx_gemm": (c_int, [c_longlong, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_longlong, c_int, c_void_p]),
        "sana_mx_linear_workspace_size": (c_size_t, [c_longlong, c_int]),
        "sana_mx_linear": (c_int, [c_longlong, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                   c_void_p, c_longlong, c_int, c_void_p, c_size_t, c_void_p]),
        "sana_sync_status": (c_int, [c_void_p]),
        "sana_selftest_bounded_wait": (c_int, [ctypes.c_uint, c_void_p]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def last_error() -> str:
    return lib.sana_last_error_string().decode()


def check(status: int):
    if status != SANA_OK:
        raise SanaError(status, last_error())


# ---------------------------------------------------------------- helpers

def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream():
    return c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SANA_BF16
    if t.dtype == torch.float32:
        return SANA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def make_shape(B, grid, heads, head_dim, t_offset=0) -> Shape:
    T, H, W = grid
    return Shape(B, T, H, W, heads, head_dim, t_offset)


class Rope:
    """Device copy of the 3D RoPE tables for frames [0, T_total) of an H x W grid."""

    def __init__(self, T_total, H, W, split, theta=10000.0, device="cuda"):
        n_t, n_h, n_w = split
        n = lib.sana_rope_tables_count(T_total, H, W, n_t, n_h, n_w)
        host = torch.empty(max(n, 1), dtype=torch.float32)
        check(lib.sana_rope_tables_host(T_total, H, W, n_t, n_h, n_w, theta, c_void_p(host.data_ptr())))
        self.host = host
        self.tables = host.to(device)
        self.struct = RopeStruct()
        check(lib.sana_rope_bind(c_void_p(self.tables.data_ptr()), T_total, H, W, n_t, n_h, n_w,
                                 ctypes.byref(self.struct)))
        self.T_total, self.H, self.W, self.split = T_total, H, W, tuple(split)


def host_rope_tables(T_total, H, W, split, theta=10000.0) -> torch.Tensor:
    """The six fp32 tables as the library computes them on the host."""
    n_t, n_h, n_w = split
    n = lib.sana_rope_tables_count(T_total, H, W, n_t, n_h, n_w)
    host = torch.empty(max(n, 1), dtype=torch.float32)
    check(lib.sana_rope_tables_host(T_total, H, W, n_t, n_h, n_w, theta, c_void_p(host.data_ptr())))
    return host[:n]


# ---------------------------------------------------------------- linear attention

def linattn_workspace_size(B, grid, heads, head_dim, dtype_code) -> int:
    s = make_shape(B, grid, heads, head_dim)
    return lib.sana_linattn_workspace_size(ctypes.byref(s), dtype_code)


def linattn_state_workspace_size(B, grid, heads, head_dim, dtype_code) -> int:
    s = make_shape(B, grid, heads, head_dim)
    return lib.sana_linattn_state_workspace_size(ctypes.byref(s), dtype_code)


def _ws(nbytes, device):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def linattn_fwd(q, k, v, gate, rope: Rope, grid, heads, eps=1e-6, out=None, ws=None):
    """Gated bidirectional ReLU linear attention with RoPE after the ReLU."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    if gate is not None:
        _need(gate, "gate")
    B, N, C = q.shape
    D = C // heads
    dt = _dtype_code(q)
    s = make_shape(B, grid, heads, D)
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = _ws(lib.sana_linattn_workspace_size(ctypes.byref(s), dt), q.device)
    check(lib.sana_linattn_fwd(ctypes.byref(s), dt, _ptr(q), _ptr(k), _ptr(v), _ptr(gate),
                               ctypes.byref(rope.struct), eps, _ptr(out), _ptr(ws), ws.numel(),
                               _stream()))
    return out


def linattn_state(k, v, rope: Rope, grid, heads, S=None, z=None, ws=None):
    """S = sum_j RoPE(phi K_j)^T V_j (B, heads, D, D) and z = sum_j phi K_j (B, heads, D), fp32."""
    _need(k, "k")
    _need(v, "v")
    B, N, C = k.shape
    D = C // heads
    dt = _dtype_code(k)
    s = make_shape(B, grid, heads, D)
    if S is None:
        S = torch.empty(B, heads, D, D, dtype=torch.float32, device=k.device)
    if z is None:
        z = torch.empty(B, heads, D, dtype=torch.float32, device=k.device)
    if ws is None:
        ws = _ws(lib.sana_linattn_state_workspace_size(ctypes.byref(s), dt), k.device)
    check(lib.sana_linattn_state(ctypes.byref(s), dt, _ptr(k), _ptr(v), ctypes.byref(rope.struct),
                                 _ptr(S), _ptr(z), _ptr(ws), ws.numel(), _stream()))
    return S, z


def linattn_apply(q, gate, rope: Rope, grid, heads, S, z, eps=1e-6, out=None):
    """Y = sigmoid(G) * RoPE(phi Q) S / (phi Q . z + eps) for a given state."""
    _need(q, "q")
    B, N, C = q.shape
    D = C // heads
    s = make_shape(B, grid, heads, D)
    if out is None:
        out = torch.empty_like(q)
    check(lib.sana_linattn_apply(ctypes.byref(s), _dtype_code(q), _ptr(q), _ptr(gate),
                                 ctypes.byref(rope.struct), _ptr(S), _ptr(z), eps, _ptr(out),
                                 _stream()))
    return out


def linattn_block_causal_step(q, k, v, gate, rope: Rope, grid, t_offset, heads, state_S, state_z,
                              commit=True, eps=1e-6, out=None, ws=None):
    """One block-causal chunk; state_S (B, heads, D, D) / state_z (B, heads, D) fp32 in place."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (state_S, "state_S"), (state_z, "state_z")):
        _need(t, n)
    B, N, C = q.shape
    D = C // heads
    dt = _dtype_code(q)
    s = make_shape(B, grid, heads, D, t_offset)
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = _ws(lib.sana_linattn_workspace_size(ctypes.byref(s), dt), q.device)
    check(lib.sana_linattn_block_causal_step(
        ctypes.byref(s), dt, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), ctypes.byref(rope.struct), eps,
        _ptr(state_S), _ptr(state_z), int(bool(commit)), _ptr(out), _ptr(ws), ws.numel(), _stream()))
    return out


def linattn_bwd(q, k, v, gate, rope: Rope, grid, heads, dy, eps=1e-6, ws=None, S=None, z=None):
    """Gradients (dq, dk, dv, dgate) of the gated linear-attention layer for dY
    (dgate is None for the ungated layer).  bf16.  S, z: the forward's state
    as linattn_state returned it for these k, v (then it is not rebuilt)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dy, "dy")):
        _need(t, n)
    if (S is None) != (z is None):
        raise ValueError("linattn_bwd: give both S and z or neither")
    B, N, C = q.shape
    D = C // heads
    dt = _dtype_code(q)
    s = make_shape(B, grid, heads, D)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg = None if gate is None else torch.empty_like(gate)
    if ws is None:
        ws = _ws(lib.sana_linattn_bwd_workspace_size(ctypes.byref(s), dt), q.device)
    if S is None:
        check(lib.sana_linattn_bwd(
            ctypes.byref(s), dt, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), ctypes.byref(rope.struct),
            eps, _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(ws), ws.numel(), _stream()))
    else:
        check(lib.sana_linattn_bwd_saved_state(
            ctypes.byref(s), dt, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), ctypes.byref(rope.struct),
            eps, _ptr(S), _ptr(z), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(ws),
            ws.numel(), _stream()))
    return dq, dk, dv, dg


def linattn_block_causal_scan_workspace_size(B, grid, heads, D, chunk_frames, dtype_code,
                                             t_offset=0) -> int:
    s = make_shape(B, grid, heads, D, t_offset)
    return lib.sana_linattn_block_causal_scan_workspace_size(ctypes.byref(s), chunk_frames,
                                                             dtype_code)


def linattn_block_causal_scan(q, k, v, gate, rope: Rope, grid, t_offset, heads, chunk_frames,
                              state_S, state_z, commit=True, eps=1e-6, out=None, ws=None):
    """A whole sequence of blocks of chunk_frames frames (the last block takes the
    remaining frames); state_S / state_z fp32 in place as for the block step."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (state_S, "state_S"), (state_z, "state_z")):
        _need(t, n)
    B, N, C = q.shape
    D = C // heads
    dt = _dtype_code(q)
    s = make_shape(B, grid, heads, D, t_offset)
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = _ws(lib.sana_linattn_block_causal_scan_workspace_size(ctypes.byref(s), chunk_frames,
                                                                   dt), q.device)
    check(lib.sana_linattn_block_causal_scan(
        ctypes.byref(s), chunk_frames, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(gate),
        ctypes.byref(rope.struct), eps, _ptr(state_S), _ptr(state_z), int(bool(commit)), _ptr(out),
        _ptr(ws), ws.numel(), _stream()))
    return out


# ---------------------------------------------------------------- anchor

def softmax_anchor_fwd(q, k, v, gate, rope, grid, heads, scale=0.0, out=None, ws=None):
    """Gated bidirectional softmax attention with 3D RoPE on Q, K (rope may be None)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    B, N, C = q.shape
    D = C // heads
    dt = _dtype_code(q)
    s = make_shape(B, grid, heads, D)
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = _ws(lib.sana_softmax_anchor_workspace_size(ctypes.byref(s), dt), q.device)
    check(lib.sana_softmax_anchor_fwd(
        ctypes.byref(s), dt, _ptr(q), _ptr(k), _ptr(v), _ptr(gate),
        None if rope is None else ctypes.byref(rope.struct), scale, _ptr(out), _ptr(ws), ws.numel(),
        _stream()))
    return out


def rope_apply(x, rope, grid, heads, mul=1.0, out=None):
    """out = mul * RoPE(x) for a (B, N, C) tensor (rope may be None: no rotation)."""
    _need(x, "x")
    B, N, C = x.shape
    s = make_shape(B, grid, heads, C // heads)
    if out is None:
        out = torch.empty_like(x)
    check(lib.sana_rope_apply(ctypes.byref(s), _dtype_code(x), _ptr(x),
                              None if rope is None else ctypes.byref(rope.struct), mul, _ptr(out),
                              _stream()))
    return out


def softmax_anchor_rotated_fwd(q_rot, k_rot, v, gate, grid, heads, out=None):
    """The anchor's attention phase on rotated operands (bf16): Q' = scale *
    log2(e) * RoPE(Q), K' = RoPE(K) as rope_apply writes them."""
    for t, n in ((q_rot, "q_rot"), (k_rot, "k_rot"), (v, "v")):
        _need(t, n)
    B, N, C = q_rot.shape
    s = make_shape(B, grid, heads, C // heads)
    if out is None:
        out = torch.empty_like(v)
    check(lib.sana_softmax_anchor_rotated_fwd(ctypes.byref(s), _ptr(q_rot), _ptr(k_rot), _ptr(v),
                                              _ptr(gate), _ptr(out), _stream()))
    return out


def anchor_tile_count(N: int) -> int:
    """Key tiles of 128 tokens; query blocks are pairs of them."""
    return (N + 127) // 128


def softmax_anchor_sparse_workspace_size(B, grid, heads, head_dim) -> int:
    s = make_shape(B, grid, heads, head_dim)
    return lib.sana_softmax_anchor_sparse_workspace_size(ctypes.byref(s), SANA_BF16)


def softmax_anchor_sparse_fwd(q, k, v, gate, rope, grid, heads, keep_tiles, tiles=None,
                              select=True, scale=0.0, out=None, ws=None):
    """Block-sparse gated softmax anchor (bf16).  With select, the library picks
    the keep_tiles key tiles of every 256-query block and writes them into
    `tiles` (allocated if None); without, the given int32 tiles
    [B, heads, n_blocks, keep_tiles] are used.  Returns (out, tiles)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    B, N, C = q.shape
    D = C // heads
    dt = _dtype_code(q)
    s = make_shape(B, grid, heads, D)
    nt = anchor_tile_count(N)
    if tiles is None:
        tiles = torch.empty(B, heads, (nt + 1) // 2, keep_tiles, dtype=torch.int32, device=q.device)
    _need(tiles, "tiles")
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = _ws(lib.sana_softmax_anchor_sparse_workspace_size(ctypes.byref(s), dt), q.device)
    check(lib.sana_softmax_anchor_sparse_fwd(
        ctypes.byref(s), dt, _ptr(q), _ptr(k), _ptr(v), _ptr(gate),
        None if rope is None else ctypes.byref(rope.struct), scale, keep_tiles, _ptr(tiles),
        int(bool(select)), _ptr(out), _ptr(ws), ws.numel(), _stream()))
    return out, tiles


# ---------------------------------------------------------------- AttnRes, norm, GEMM

def attnres_route(sources, w, rms_eps=1e-6, out=None, alpha=None, want_alpha=False):
    """h = sum_i softmax_i(w . RMSNorm(v_i)) v_i over (B, N, C) sources."""
    for i, t in enumerate(sources):
        _need(t, f"sources[{i}]")
    _need(w, "w")
    B, N, C = sources[0].shape
    dt = _dtype_code(sources[0])
    if out is None:
        out = torch.empty_like(sources[0])
    if want_alpha and alpha is None:
        alpha = torch.empty(B, N, len(sources), dtype=torch.float32, device=sources[0].device)
    arr = (c_void_p * len(sources))(*[t.data_ptr() for t in sources])
    check(lib.sana_attnres_route(B, N, C, dt, arr, len(sources), _ptr(w), rms_eps, _ptr(out),
                                 _ptr(alpha), _stream()))
    return (out, alpha) if want_alpha else out


def attnres_route_bwd(sources, w, dh, rms_eps=1e-6, ws=None):
    """Gradients (list of d sources, d w) of attnres_route for dh.  bf16 sources."""
    for i, t in enumerate(sources):
        _need(t, f"sources[{i}]")
    _need(w, "w")
    _need(dh, "dh")
    B, N, C = sources[0].shape
    dt = _dtype_code(sources[0])
    grads = [torch.empty_like(t) for t in sources]
    dw = torch.empty(C, dtype=torch.float32, device=w.device)
    if ws is None:
        ws = _ws(lib.sana_attnres_route_bwd_workspace_size(B, N, C), w.device)
    src = (c_void_p * len(sources))(*[t.data_ptr() for t in sources])
    dst = (c_void_p * len(grads))(*[t.data_ptr() for t in grads])
    check(lib.sana_attnres_route_bwd(B, N, C, dt, src, len(sources), _ptr(w), rms_eps, _ptr(dh),
                                     dst, _ptr(dw), _ptr(ws), ws.numel(), _stream()))
    return grads, dw


def rmsnorm(x, eps=1e-6, out=None):
    _need(x, "x")
    C = x.shape[-1]
    rows = x.numel() // C
    if out is None:
        out = torch.empty_like(x)
    check(lib.sana_rmsnorm(rows, C, _dtype_code(x), _ptr(x), eps, _ptr(out), _stream()))
    return out


def gemm_bf16(A, W, out=None, epilogue=EPI_NONE):
    """out = epilogue(A . W^T), A (M, K) bf16, W (N, K) bf16, fp32 accumulation."""
    M, K = A.shape[-2] if A.dim() == 2 else A.numel() // A.shape[-1], A.shape[-1]
    N = W.shape[0]
    if out is None:
        out = torch.empty(*A.shape[:-1], N, dtype=torch.bfloat16, device=A.device)
    check(lib.sana_gemm_bf16(M, N, K, _ptr(A), A.stride(-2) if A.dim() >= 2 else K, _ptr(W),
                             _ptr(out), out.stride(-2) if out.dim() >= 2 else N, epilogue, _stream()))
    return out


# ---------------------------------------------------------------- stack

def stack_config(layers, block_span=8, ratio=4, use_attnres=True, ffn_mult=3, eps=1e-6,
                 rms_eps=1e-6, anchor_scale=0.0, anchor_keep_tiles=0,
                 mx_projections=False) -> StackConfig:
    return StackConfig(layers, block_span, ratio, int(bool(use_attnres)), ffn_mult, eps, rms_eps,
                       anchor_scale, anchor_keep_tiles, int(bool(mx_projections)))


def mx_quantize_stack_weights(weights):
    """Per-layer weight dicts with the MX form of every projection weight added
    (keys '<name>_mxq' codes and '<name>_mxs' scales), as the stack reads them
    with mx_projections on."""
    out = []
    for d in weights:
        e = dict(d)
        for key in ("qkvg", "o", "up", "down"):
            if key in d:
                e[key + "_mxq"], e[key + "_mxs"] = mx_quantize(d[key], fp4=True)
        out.append(e)
    return out


def hybrid_stack_fwd(x, weights, w_attn, w_ffn, rope: Rope, grid, heads, cfg: StackConfig,
                     out=None, ws=None):
    _need(x, "x")
    B, N, C = x.shape
    s = make_shape(B, grid, heads, C // heads)
    L = cfg.layers

    def arr(key):
        if cfg.ffn_mult == 0 and key.split("_")[0] in ("up", "down"):
            return None
        if any(key not in weights[l] for l in range(L)):
            return None
        return (c_void_p * L)(*[weights[l][key].data_ptr() for l in range(L)])

    names = ("qkvg", "o", "up", "down")
    keep = {k: arr(k) for k in names + tuple(n + sfx for n in names for sfx in ("_mxq", "_mxs"))}
    p = lambda a: None if a is None else ctypes.cast(a, POINTER(c_void_p))
    sw = StackWeights(
        p(keep["qkvg"]), p(keep["o"]), p(keep["up"]), p(keep["down"]),
        None if w_attn is None else w_attn.data_ptr(), None if w_ffn is None else w_ffn.data_ptr(),
        p(keep["qkvg_mxq"]), p(keep["qkvg_mxs"]), p(keep["o_mxq"]), p(keep["o_mxs"]),
        p(keep["up_mxq"]), p(keep["up_mxs"]), p(keep["down_mxq"]), p(keep["down_mxs"]))
    if out is None:
        out = torch.empty_like(x)
    if ws is None:
        ws = _ws(lib.sana_hybrid_stack_workspace_size(ctypes.byref(s), ctypes.byref(cfg)), x.device)
    check(lib.sana_hybrid_stack_fwd(ctypes.byref(s), ctypes.byref(cfg), ctypes.byref(sw),
                                    ctypes.byref(rope.struct), _ptr(x), _ptr(out), _ptr(ws),
                                    ws.numel(), _stream()))
    return out


def hybrid_stack_workspace_size(B, grid, heads, cfg: StackConfig, head_dim=128) -> int:
    s = make_shape(B, grid, heads, head_dim)
    return lib.sana_hybrid_stack_workspace_size(ctypes.byref(s), ctypes.byref(cfg))


def hybrid_stack_workspace_views(ws, B, grid, heads, cfg: StackConfig, head_dim=128) -> dict:
    """Views of the stack's intermediates inside its workspace `ws` (a uint8
    tensor) after a call: keys x_hat, q, k, v, g, attn, ffn (absent when
    ffn_mult is 0) and blocks (list), each (B, N, width) bf16."""
    s = make_shape(B, grid, heads, head_dim)
    lay = StackWsLayout()
    check(lib.sana_hybrid_stack_workspace_layout(ctypes.byref(s), ctypes.byref(cfg),
                                                 ctypes.byref(lay)))
    N = grid[0] * grid[1] * grid[2]
    C = heads * head_dim

    def view(off, width):
        nbytes = B * N * width * 2
        return ws[off:off + nbytes].view(torch.bfloat16).view(B, N, width)

    out = {k: view(getattr(lay, k), C) for k in ("x_hat", "q", "k", "v", "g", "attn")}
    if cfg.ffn_mult > 0:
        out["ffn"] = view(lay.ffn, cfg.ffn_mult * C)
    out["blocks"] = [view(lay.blocks[i], C) for i in range(lay.num_blocks)]
    return out


# ---------------------------------------------------------------- MX projection GEMM

def mx_quantize(x, fp4=False):
    """MX quantisation of a bf16 (rows, K) tensor along K: returns (codes,
    scales) as uint8 tensors -- E4M3 codes (rows, K), or E2M1 codes packed two
    per byte (rows, K/2) with fp4, and the E8M0 scale atoms."""
    _need(x, "x")
    K = x.shape[-1]
    rows = x.numel() // K
    q = torch.empty(rows, K // 2 if fp4 else K, dtype=torch.uint8, device=x.device)
    sf = torch.empty(max(int(lib.sana_mx_scale_bytes(rows, K)), 16), dtype=torch.uint8,
                     device=x.device)
    check(lib.sana_mx_quantize(_ptr(x), rows, K, int(bool(fp4)), _ptr(q), _ptr(sf), _stream()))
    return q, sf


def mx_gemm(xq, x_scales, wq, w_scales, N, out=None, epilogue=EPI_NONE):
    """out = epilogue(Q8(x) . Q4(w)^T) from quantised operands (see mx_quantize)."""
    M, K = xq.shape
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=xq.device)
    check(lib.sana_mx_gemm(M, N, K, _ptr(xq), _ptr(x_scales), _ptr(wq), _ptr(w_scales), _ptr(out),
                           out.stride(0), epilogue, _stream()))
    return out


def mx_linear(x, wq, w_scales, N, out=None, epilogue=EPI_NONE, ws=None):
    """The quantised projection of bf16 activations x (M, K) against
    pre-quantised MXFP4 weights: activations quantised to MXFP8 on the fly."""
    _need(x, "x")
    M, K = x.shape
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = _ws(lib.sana_mx_linear_workspace_size(M, K), x.device)
    check(lib.sana_mx_linear(M, N, K, _ptr(x), _ptr(wq), _ptr(w_scales), _ptr(out), out.stride(0),
                             epilogue, _ptr(ws), ws.numel(), _stream()))
    return out


def selftest_bounded_wait(limit_ms=50):
    """Enqueue a kernel whose bounded wait runs out (see include/sana.h)."""
    check(lib.sana_selftest_bounded_wait(limit_ms, _stream()))


def sync_status():
    check(lib.sana_sync_status(_stream()))
