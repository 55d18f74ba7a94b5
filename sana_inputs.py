"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle runs.

This module holds no arithmetic of the method: it only draws numbers and
rounds them to the storage dtype.  Recipe: numpy ``Generator(PCG64(seed))``,
``standard_normal`` in float32, times a scale, rounded to bf16 with
round-to-nearest-even (torch's float32 -> bfloat16 cast) where the workload
is bf16.  Seeds: seed = 1000 * config + tensor_id with tensor ids Q=1, K=2,
V=3, G (or X) = 4, projection weights 100 + 10 * layer + {0: qkvg, 1: o,
2: up, 3: down}, router queries 20/21,
AttnRes sources 30 + i.  Block-causal chunks use
seed = 100000 * config + 100 * chunk + tensor_id (no overlap with the
per-config seeds).

The workload shapes are latent token grids of video clips (token n =
(t * H + h) * W + w):

* tiny: T=2, H=4, W=4 (N=32), 2 heads, D=16, fp32;
* 480p: T=21, H=30, W=52 (N=32,760), 24 heads, D=128, bf16;
* 720p/5s: T=21, H=45, W=80 (N=75,600), 24 heads, D=128, bf16;
* 720p/60s block-causal: T=241, H=45, W=80 in chunks of 3 frames;
* the 16-layer stack on the 720p/5s grid with hidden size 3072.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    config: int
    B: int
    T: int
    H: int
    W: int
    heads: int
    D: int
    dtype: str            # "f32" or "bf16"
    rope_split: tuple     # rotary pairs over (t, h, w)
    chunk_frames: int = 0  # block-causal chunk length in latent frames

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def C(self) -> int:
        return self.heads * self.D

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


TINY = Workload("tiny", 1, 1, 2, 4, 4, 2, 16, "f32", (2, 3, 3))
P480 = Workload("480p", 2, 1, 21, 30, 52, 24, 128, "bf16", (22, 21, 21))
P720 = Workload("720p", 3, 1, 21, 45, 80, 24, 128, "bf16", (22, 21, 21))
LONG = Workload("720p60s_causal", 4, 1, 241, 45, 80, 24, 128, "bf16", (22, 21, 21),
                chunk_frames=3)
STACK = Workload("720p_stack", 5, 1, 21, 45, 80, 24, 128, "bf16", (22, 21, 21))

WORKLOADS = {w.name: w for w in (TINY, P480, P720, LONG, STACK)}

Q_ID, K_ID, V_ID, G_ID = 1, 2, 3, 4


def seed_of(config: int, tensor_id: int, chunk: int | None = None) -> int:
    if chunk is None:
        return 1000 * config + tensor_id
    return 100000 * config + 100 * chunk + tensor_id


def normal(seed: int, shape, dtype=torch.bfloat16, scale: float = 1.0) -> torch.Tensor:
    """Seeded N(0, scale^2) draws, rounded to ``dtype`` (CPU tensor)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(size=tuple(shape), dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    t = torch.from_numpy(x)
    if dtype != torch.float32:
        t = t.to(dtype)
    return t


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a (CPU or device) tensor for the oracle."""
    return t.detach().to("cpu", torch.float64).numpy()


def qkvg(wl: Workload, gate: bool = True, B: int | None = None, N: int | None = None,
         chunk: int | None = None):
    """Q, K, V (and gate logits G) of shape (B, N, C) for a workload."""
    B = wl.B if B is None else B
    N = wl.N if N is None else N
    shape = (B, N, wl.C)
    out = [normal(seed_of(wl.config, i, chunk), shape, wl.torch_dtype)
           for i in (Q_ID, K_ID, V_ID)]
    out.append(normal(seed_of(wl.config, G_ID, chunk), shape, wl.torch_dtype)
               if gate else None)
    return tuple(out)


def chunk_frames(wl: Workload):
    """Partition of wl.T frames into block-causal chunks: full chunks of
    wl.chunk_frames frames, then one shorter final chunk if T does not divide
    (241 = 80 * 3 + 1).  Returns a list of (t_offset, frames)."""
    out = []
    t = 0
    while t < wl.T:
        f = min(wl.chunk_frames, wl.T - t)
        out.append((t, f))
        t += f
    return out


def causal_chunk(wl: Workload, chunk: int, frames: int):
    """Q, K, V of one block-causal chunk, (B, frames*H*W, C)."""
    shape = (wl.B, frames * wl.H * wl.W, wl.C)
    return tuple(normal(seed_of(wl.config, i, chunk), shape, wl.torch_dtype)
                 for i in (Q_ID, K_ID, V_ID))


def projection_weights(config: int, layers: int, C: int, ffn_mult: int,
                       dtype=torch.bfloat16):
    """Per-layer projection weights (out, in) ~ N(0, 1/fan_in)."""
    ws = []
    for l in range(layers):
        base = 100 + 10 * l
        d = {
            "qkvg": normal(seed_of(config, base + 0), (4 * C, C), dtype, C ** -0.5),
            "o": normal(seed_of(config, base + 1), (C, C), dtype, C ** -0.5),
        }
        if ffn_mult:
            F = ffn_mult * C
            d["up"] = normal(seed_of(config, base + 2), (F, C), dtype, C ** -0.5)
            d["down"] = normal(seed_of(config, base + 3), (C, F), dtype, F ** -0.5)
        ws.append(d)
    return ws


def router_queries(config: int, C: int):
    """Shared AttnRes router queries (attention, FFN) ~ N(0, 1/C), fp32."""
    return (normal(seed_of(config, 20), (C,), torch.float32, C ** -0.5),
            normal(seed_of(config, 21), (C,), torch.float32, C ** -0.5))


def attnres_sources(config: int, S: int, B: int, N: int, C: int, dtype=torch.bfloat16):
    """S AttnRes sources (embedding, summaries, partial sum) ~ N(0, 1)."""
    return [normal(seed_of(config, 30 + i), (B, N, C), dtype) for i in range(S)]
