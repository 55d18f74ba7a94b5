#!/usr/bin/env python
"""Benchmark of the gated ReLU-RoPE linear-attention layer at the 720p/5s
latent shape (B=1, T=21, H=45, W=80 -> N=75,600 tokens, 24 heads, D=128,
bf16, sigmoid output gate) on B200, through libsana's C ABI.

One step = one sana_linattn_fwd call: ReLU + RoPE of K, the N-axis state
reduction S = sum RoPE(phi K)^T V and z = sum phi K, the fixed-order combine,
ReLU + RoPE of Q, the numerator Q'S, the RoPE-free denominator, and the
sigmoid gate.  Inputs (4 x 464.5 MB) exceed the 126 MB L2, so no flush is
needed between steps.

`value` is whole-job tokens/s (all ranks; each rank runs its own layer, weak
scaling), device-timed with CUDA events, max over ranks.  Rank 0 prints one
JSON line.  `--impl reference` times the float64 CPU oracle instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import sana_inputs as si  # noqa: E402

METRIC = "linear-attn tokens/s and TFLOP/s per layer @720p/5s bf16; % of roofline"
WL = si.P720
TENSOR_BYTES = WL.B * WL.N * WL.C * 2                  # one (B, N, C) bf16 tensor
LAYER_BYTES = 5 * TENSOR_BYTES                         # Q, K, V, G read; Y written
APPLY_BYTES = 3 * TENSOR_BYTES                         # output kernel: Q, G read; Y written
LAYER_FLOPS = 4 * WL.B * WL.N * WL.heads * WL.D ** 2   # K'^T V and Q' S
FALLBACK_HBM_GBS = 6650.0


FALLBACK_BF16_TFLOPS = 1590.0
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 tensor peak (burst: the anchor is timed on its own)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if "bf16_tflops" in d:
            return d["bf16_tflops"], "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def tensor_peak_sustained():
    """Dense bf16 tensor peak held for seconds under the power cap, or None."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return json.load(open(p)).get("bf16_tflops_sustained")
    return None


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("linattn_tc.cu", "sana_common.cuh", "rope_dev.cuh", "pdl.cuh"):
        h.update(open(os.path.join(ROOT, "softmax_attention_sana_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the output kernel from the committed ncu summary,
    if it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "linattn_out_kernel_720p.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m_h = re.search(r"kernel source hash:\s*`?([0-9a-f]{16})", txt)
    m_t = re.search(r"dram bytes per launch:\s*`?([0-9.eE+]+)", txt)
    if not (m_h and m_t) or m_h.group(1) != kernel_source_hash():
        return None
    return float(m_t.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """Largest value over all ranks (device tensor under NCCL, host under gloo)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, ms_per_step_local, world):
    """Whole-job throughput: the units all ranks processed per step divided by
    the slowest rank's time per step (weak scaling: every rank has its own
    layer).  Returns (units per second, ms per step of the slowest rank)."""
    ms = max_over_ranks(ms_per_step_local, world)
    return world * units_per_rank / (ms / 1e3), ms


def time_loop(fn, steps):
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    for _ in range(steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps  # ms


# ---------------------------------------------------------------- CPU oracle leg

_ORACLE_INPUTS = {}


def oracle_inputs(heads, cpu_tensors=None):
    """float64 copies of the first `heads` heads of the 720p layer's inputs."""
    if heads not in _ORACLE_INPUTS:
        ts = cpu_tensors if cpu_tensors is not None else si.qkvg(WL)
        cols = slice(0, heads * WL.D)
        _ORACLE_INPUTS[heads] = tuple(si.as_f64(t[..., cols]) for t in ts)
    return _ORACLE_INPUTS[heads]


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # pragma: no cover
        return os.cpu_count()


def oracle_sample(heads, n_tok, cpu_tensors=None):
    """Time the float64 oracle on `heads` heads and the first `n_tok` tokens of
    the 720p layer (state over those tokens, then their outputs).  The oracle's
    work is linear in heads x tokens, so the time scales to a whole layer by
    (24 / heads) x (N / n_tok).  Returns (tokens/s of a layer, seconds, text)."""
    from oracle import sana_oracle as orc
    q, k, v, g = (t[:, :n_tok] for t in oracle_inputs(heads, cpu_tensors))
    t0 = time.perf_counter()
    ang = orc.rope_angles(WL.T, WL.H, WL.W, *WL.rope_split)[:n_tok]
    S, z = orc.linattn_state(k, v, ang, heads)
    orc.linattn_apply(q, S, z, ang, heads, gate=g)
    dt = time.perf_counter() - t0
    scale = (WL.heads / heads) * (WL.N / n_tok)
    desc = (f"oracle (numpy float64) on {heads} of {WL.heads} heads x {n_tok} of {WL.N} tokens "
            f"of the 720p layer, time scaled x{scale:.2f} to a whole layer")
    return WL.B * WL.N / (dt * scale), dt, desc


def run_reference(args, world, rank):
    if rank != 0:
        return
    # calibrate the per-(head, token) cost, then size each step's sample so the
    # whole --steps/--warmup run takes about args.ref_budget seconds
    _, dt, _ = oracle_sample(1, 4096)
    _, dt, _ = oracle_sample(1, 4096)
    per_tok = dt / 4096
    budget = max(0.02, min(5.0, args.ref_budget / (args.steps + args.warmup)))
    n_tok = int(min(WL.N, max(512, budget / per_tok)))
    for _ in range(args.warmup):
        oracle_sample(1, n_tok)
    vals, secs = [], []
    desc = ""
    for _ in range(args.steps):
        v, dt, desc = oracle_sample(1, n_tok)
        vals.append(v)
        secs.append(dt)
    value = float(np.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * float(np.median(secs)),
        "ms_per_step_kind": "measured: wall time of one step's bounded sample (1 head x "
                            f"{n_tok} tokens); value is that sample's rate scaled to a whole layer",
        "extrapolated_ms_per_layer": 1e3 * WL.B * WL.N / value,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": desc + " (median over steps)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config():
    return {"workload": "720p/5s gated linear-attention layer", "B": WL.B, "T": WL.T, "H": WL.H,
            "W": WL.W, "N": WL.N, "heads": WL.heads, "head_dim": WL.D, "gate": "sigmoid",
            "rope_split": list(WL.rope_split),
            "l2": "no flush: 4 inputs x 464.5 MB per step exceed the 126 MB L2"}


# ---------------------------------------------------------------- GPU leg

def components(sana, args):
    """Other rows of the hot path, each timed on its own with CUDA events."""
    out = {}
    # 480p layer
    wl = si.P480
    q, k, v, g = (t.cuda() for t in si.qkvg(wl))
    rope = sana.Rope(wl.T, wl.H, wl.W, wl.rope_split)
    ws = torch.empty(sana.linattn_workspace_size(wl.B, (wl.T, wl.H, wl.W), wl.heads, wl.D, 1),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty_like(q)
    f = lambda: sana.linattn_fwd(q, k, v, g, rope, (wl.T, wl.H, wl.W), wl.heads, out=y, ws=ws)
    for _ in range(5):
        f()
    ms = time_loop(f, 50)
    out["linattn_480p"] = {"ms": ms, "tokens_per_s": wl.N / (ms / 1e3),
                           "GB_per_s": 5 * wl.N * wl.C * 2 / (ms / 1e3) / 1e9}
    del q, k, v, g, y
    # block-causal chunk step (720p/60s chunk: 3 frames, 10,800 tokens, state carried)
    ms_b2b, ms_iso, nb = chunk_step_times()
    out["causal_chunk_720p60s"] = {
        "ms": ms_b2b, "tokens_per_s": 10800 / (ms_b2b / 1e3), "GB_per_s": nb / (ms_b2b / 1e3) / 1e9,
        "frac_of_hbm_peak": nb / (ms_b2b / 1e3) / 1e9 / peaks()[0],
        "timing": "device time per step, 64 steps back to back over 4 distinct chunks (1.06 GB of "
                  "inputs > L2)",
        "isolated_ms": ms_iso,
        "isolated": "one call between L2 flushes, from the Python call to the last kernel "
                    "(includes the host's argument marshalling and launches)"}
    # the whole 720p/60s sequence through the block-causal scan (80 blocks of
    # 3 frames + 1 frame, 867,600 tokens; inputs drawn on the device: 16 GB)
    wl = si.LONG
    step_ms = ms_b2b
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4000)
    shape = (1, wl.N, wl.C)
    q, k, v = (torch.randn(shape, generator=gen, device="cuda", dtype=torch.bfloat16)
               for _ in range(3))
    rope = sana.Rope(wl.T, wl.H, wl.W, wl.rope_split)
    S = torch.zeros(1, wl.heads, wl.D, wl.D, device="cuda")
    z = torch.zeros(1, wl.heads, wl.D, device="cuda")
    ws = torch.empty(sana.linattn_block_causal_scan_workspace_size(1, (wl.T, wl.H, wl.W), wl.heads,
                                                                   wl.D, 3, 1),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty_like(q)
    f = lambda: sana.linattn_block_causal_scan(q, k, v, None, rope, (wl.T, wl.H, wl.W), 0,
                                               wl.heads, 3, S, z, commit=False, out=y, ws=ws)
    for _ in range(3):
        f()
    ms = time_loop(f, 10)
    nb = 4 * wl.N * wl.C * 2 + 2 * wl.heads * (wl.D * wl.D + wl.D) * 4
    nchunks = len(si.chunk_frames(wl))
    out["causal_scan_720p60s"] = {
        "ms": ms, "tokens_per_s": wl.N / (ms / 1e3), "GB_per_s": nb / (ms / 1e3) / 1e9,
        "frac_of_hbm_peak": nb / (ms / 1e3) / 1e9 / peaks()[0],
        "vs_chunk_steps": f"{nchunks} steps x {step_ms:.3f} ms = {nchunks * step_ms:.2f} ms",
        "l2": "no flush: 16 GB of inputs per call"}
    del q, k, v, y, ws
    # AttnRes route over 3 sources at 720p/5s
    srcs = [t.cuda() for t in si.attnres_sources(5, 3, 1, si.P720.N, si.P720.C)]
    w_attn, _ = (t.cuda() for t in si.router_queries(5, si.P720.C))
    h = torch.empty_like(srcs[0])
    f = lambda: sana.attnres_route(srcs, w_attn, out=h)
    for _ in range(3):
        f()
    ms = time_loop(f, 20)
    out["attnres_route_720p_3src"] = {"ms": ms, "GB_per_s": 4 * TENSOR_BYTES / (ms / 1e3) / 1e9}
    # its backward: 3 sources and dh read, 3 source gradients written, dw summed
    dh = si.normal(7100, (1, si.P720.N, si.P720.C)).cuda()
    wsb = torch.empty(sana._lib.lib.sana_attnres_route_bwd_workspace_size(1, si.P720.N, si.P720.C),
                      dtype=torch.uint8, device="cuda")
    f = lambda: sana.attnres_route_bwd(srcs, w_attn, dh, ws=wsb)
    for _ in range(3):
        f()
    ms = time_loop(f, 20)
    out["attnres_route_bwd_720p_3src"] = {"ms": ms, "GB_per_s": 7 * TENSOR_BYTES / (ms / 1e3) / 1e9}
    del srcs, h, dh, wsb
    # backward of the gated linear-attention layer (S, z recomputed)
    q, k, v, g = (t.cuda() for t in si.qkvg(WL))
    dy = si.normal(7000, (1, WL.N, WL.C)).cuda()
    rope = sana.Rope(WL.T, WL.H, WL.W, WL.rope_split)
    f = lambda: sana.linattn_bwd(q, k, v, g, rope, (WL.T, WL.H, WL.W), WL.heads, dy)
    for _ in range(3):
        f()
    ms = time_loop(f, 20)
    out["linattn_bwd_720p"] = {"ms": ms, "tokens_per_s": WL.N / (ms / 1e3),
                               "GB_per_s": 9 * TENSOR_BYTES / (ms / 1e3) / 1e9}
    # the same backward given the forward's state (k, v not read a second time)
    S, z = sana.linattn_state(k, v, rope, (WL.T, WL.H, WL.W), WL.heads)
    f = lambda: sana.linattn_bwd(q, k, v, g, rope, (WL.T, WL.H, WL.W), WL.heads, dy, S=S, z=z)
    for _ in range(3):
        f()
    ms = time_loop(f, 20)
    out["linattn_bwd_saved_state_720p"] = {"ms": ms, "tokens_per_s": WL.N / (ms / 1e3),
                                           "GB_per_s": 9 * TENSOR_BYTES / (ms / 1e3) / 1e9}
    del q, k, v, g, dy, S, z
    # projection GEMM of the stack: QKVG at 720p, (75,600 x 3072) . (12,288 x 3072)^T
    A = torch.randn(WL.N, WL.C, device="cuda", dtype=torch.bfloat16)
    Wq = torch.randn(4 * WL.C, WL.C, device="cuda", dtype=torch.bfloat16) * WL.C ** -0.5
    Yq = torch.empty(WL.N, 4 * WL.C, device="cuda", dtype=torch.bfloat16)
    f = lambda: sana.gemm_bf16(A, Wq, out=Yq)
    for _ in range(3):
        f()
    ms = time_loop(f, 10)
    out["gemm_qkvg_720p"] = {"ms": ms, "TFLOP_per_s": 2 * WL.N * 4 * WL.C * WL.C / (ms / 1e3) / 1e12}
    bf16_ms = ms
    # the same projection quantised: MXFP4 weights (quantised once, untimed),
    # MXFP8 activations quantised on the fly (sana_mx_linear), and the
    # block-scaled GEMM alone on pre-quantised activations
    try:
        wq, wsc = sana.mx_quantize(Wq, fp4=True)
        xq, xs = sana.mx_quantize(A)
        ws_mx = torch.empty(sana._lib.lib.sana_mx_linear_workspace_size(WL.N, WL.C),
                            dtype=torch.uint8, device="cuda")
        g = lambda: sana.mx_gemm(xq, xs, wq, wsc, 4 * WL.C, out=Yq)
        for _ in range(3):
            g()
        ms_g = time_loop(g, 10)
        f = lambda: sana.mx_linear(A, wq, wsc, 4 * WL.C, out=Yq, ws=ws_mx)
        for _ in range(3):
            f()
        ms = time_loop(f, 10)
        q = lambda: sana.mx_quantize(A)
        ms_q = time_loop(q, 10)
        flops = 2 * WL.N * 4 * WL.C * WL.C
        out["mx_linear_qkvg_720p"] = {
            "ms": ms, "TFLOP_per_s": flops / (ms / 1e3) / 1e12, "vs_bf16_gemm": bf16_ms / ms,
            "gemm_ms": ms_g, "gemm_TFLOP_per_s": flops / (ms_g / 1e3) / 1e12,
            "frac_of_nominal_fp8_peak": flops / (ms_g / 1e3) / 1e12 / (2 * SPEC_BF16_TFLOPS),
            "activation_quantise_ms": ms_q,
            "activation_quantise_GB_per_s": (WL.N * WL.C * 3 + WL.N * WL.C / 32) / (ms_q / 1e3) / 1e9}
        del wq, wsc, xq, xs, ws_mx
    except Exception as e:  # keep the rest of the line if this row fails
        out["mx_linear_qkvg_720p"] = {"unavailable": str(e)[:200]}
    del A, Wq, Yq
    # softmax anchor at 720p/5s
    if args.no_anchor:
        out["softmax_anchor_720p"] = {"skipped": "--no-anchor"}
        return out
    try:
        grid = (WL.T, WL.H, WL.W)
        q, k, v, g = (t.cuda() for t in si.qkvg(WL))
        rope = sana.Rope(WL.T, WL.H, WL.W, WL.rope_split)
        ws = torch.empty(int(4 * TENSOR_BYTES // 2 + (1 << 20)), dtype=torch.uint8, device="cuda")
        y = torch.empty_like(q)
        flops = 4 * WL.N * WL.N * WL.heads * WL.D
        # phase 1: the RoPE prepass (Q and K rotated, Q scaled by scale * log2 e)
        qr, kr = torch.empty_like(q), torch.empty_like(k)
        mul = WL.D ** -0.5 * 1.4426950408889634
        pre = lambda: (sana.rope_apply(q, rope, grid, WL.heads, mul=mul, out=qr),
                       sana.rope_apply(k, rope, grid, WL.heads, out=kr))
        for _ in range(3):
            pre()
        ms_pre = time_loop(pre, 20)
        out["anchor_rope_prepass_720p"] = {
            "ms": ms_pre, "launches": 2, "GB_per_s": 4 * TENSOR_BYTES / (ms_pre / 1e3) / 1e9,
            "frac_of_hbm_peak": 4 * TENSOR_BYTES / (ms_pre / 1e3) / 1e9 / peaks()[0],
            "algorithmic_bytes": 4 * TENSOR_BYTES, "l2": "no flush: 4 x 464.5 MB per call"}
        # phase 2: the attention kernel alone on the rotated operands
        att = lambda: sana.softmax_anchor_rotated_fwd(qr, kr, v, g, grid, WL.heads, out=y)
        att()
        ms_att = time_loop(att, 3)
        tp, tp_kind = tensor_peak()
        ach = flops / (ms_att / 1e3) / 1e12
        out["anchor_kernel_720p"] = {"ms": ms_att, "TFLOP_per_s": ach}
        anchor_roof = {"bound": "tensor", "kernel": "anchor_kernel (QK^T, softmax, PV; 720p/5s)",
                       "achieved": ach, "peak": tp, "unit": "TFLOP/s", "frac": ach / tp,
                       "peak_kind": tp_kind + " burst (cuBLAS bf16)", "spec_peak": SPEC_BF16_TFLOPS,
                       "spec_frac": ach / SPEC_BF16_TFLOPS, "traffic": None,
                       "algorithmic_flops_per_launch": flops, "ms_per_launch": ms_att}
        sus = tensor_peak_sustained()
        if sus:  # context: the same GEMM held for seconds under the power cap
            anchor_roof["sustained_peak"] = sus
            anchor_roof["sustained_frac"] = ach / sus
        out["_anchor_roofline"] = anchor_roof
        # the whole call (prepass + kernel)
        f = lambda: sana.softmax_anchor_fwd(q, k, v, g, rope, grid, WL.heads, out=y, ws=ws)
        f()
        ms = time_loop(f, 3)
        out["softmax_anchor_720p"] = {"ms": ms, "TFLOP_per_s": flops / (ms / 1e3) / 1e12,
                                      "frac_of_spec_roofline": (flops / SPEC_BF16_TFLOPS / 1e12 * 1e3) / ms}
        dense_ms = ms
        del qr, kr
        # block-sparse anchor: each 256-query block keeps a quarter of the 591
        # key tiles (selection by pooled logits included in the timing)
        nkt = sana.anchor_tile_count(WL.N)
        keep = (nkt + 3) // 4
        ws = torch.empty(sana.softmax_anchor_sparse_workspace_size(1, (WL.T, WL.H, WL.W), WL.heads,
                                                                   WL.D),
                         dtype=torch.uint8, device="cuda")
        tiles = torch.empty(1, WL.heads, (nkt + 1) // 2, keep, dtype=torch.int32, device="cuda")
        f = lambda: sana.softmax_anchor_sparse_fwd(q, k, v, g, rope, (WL.T, WL.H, WL.W), WL.heads,
                                                   keep, tiles=tiles, out=y, ws=ws)
        f()
        ms = time_loop(f, 5)
        kept = 4 * WL.N * min(WL.N, keep * 128) * WL.heads * WL.D
        out["softmax_anchor_sparse_720p_25pct"] = {
            "ms": ms, "keep_tiles": keep, "key_tiles": nkt,
            "TFLOP_per_s_executed": kept / (ms / 1e3) / 1e12,
            "speedup_vs_dense": dense_ms / ms}
        del q, k, v, g, y, ws, tiles
    except Exception as e:  # not built yet
        out["softmax_anchor_720p"] = {"unavailable": str(e)[:200]}
    # whole stacks on the 720p/5s grid: the 4-layer 3:1 group (no AttnRes, no
    # FFN), the same with block-sparse anchors, and the 16-layer AttnRes stack
    # with FFN 3C (weights drawn on the device, N(0, 1/fan_in))
    if not args.no_stacks:
        grid = (WL.T, WL.H, WL.W)
        rope = sana.Rope(WL.T, WL.H, WL.W, WL.rope_split)
        keep = (sana.anchor_tile_count(WL.N) + 3) // 4
        for name, layers, attnres, ffn, kt, mx in (
                ("stack_720p_group4", 4, False, 0, 0, False),
                ("stack_720p_group4_sparse25", 4, False, 0, keep, False),
                ("stack_720p_attnres16", 16, True, 3, 0, False),
                ("stack_720p_attnres16_mx", 16, True, 3, 0, True)):
            gen = torch.Generator(device="cuda")
            gen.manual_seed(5000 + layers)
            rn = lambda *sh, sc=1.0: (torch.randn(sh, generator=gen, device="cuda") * sc).to(
                torch.bfloat16)
            x = rn(1, WL.N, WL.C)
            C, F = WL.C, ffn * WL.C
            ws_l = []
            for _ in range(layers):
                d = {"qkvg": rn(4 * C, C, sc=C ** -0.5), "o": rn(C, C, sc=C ** -0.5)}
                if ffn:
                    d["up"], d["down"] = rn(F, C, sc=C ** -0.5), rn(C, F, sc=F ** -0.5)
                ws_l.append(d)
            w_attn, w_ffn = (t.cuda() for t in si.router_queries(5, WL.C))
            cfg = sana.stack_config(layers, block_span=8, use_attnres=attnres, ffn_mult=ffn,
                                    anchor_keep_tiles=kt, mx_projections=mx)
            if mx:  # MXFP4 weights quantised once, outside the timing
                ws_l = sana.mx_quantize_stack_weights(ws_l)
            y = torch.empty_like(x)
            f = lambda: sana.hybrid_stack_fwd(x, ws_l, w_attn, w_ffn, rope, grid, WL.heads, cfg, out=y)
            f()
            ms = time_loop(f, 2)
            nan = 4 * WL.N * WL.N * WL.heads * WL.D
            lin = 4 * WL.N * WL.heads * WL.D ** 2
            proj = 2 * WL.N * WL.C * WL.C * (4 + 1 + 2 * ffn)
            nanc = layers // 4
            if kt:  # executed anchor work of the kept tiles
                nan = 4 * WL.N * min(WL.N, kt * 128) * WL.heads * WL.D
            flops = nanc * nan + (layers - nanc) * lin + layers * proj
            tp, tp_kind = tensor_peak()
            out[name] = {"ms": ms, "TFLOP_per_s": flops / (ms / 1e3) / 1e12, "layers": layers,
                         "attnres": attnres, "ffn_mult": ffn, "flops": flops,
                         "frac_of_tensor_peak": flops / (ms / 1e3) / 1e12 / tp,
                         "frac_of_spec_tensor_peak": flops / (ms / 1e3) / 1e12 / SPEC_BF16_TFLOPS,
                         "timing": "2 calls after 1 warm-up, CUDA events"}
            if kt:
                out[name]["anchor_keep_tiles"] = kt
            if mx:
                out[name]["projections"] = ("MXFP8 activations x MXFP4 weights (flops counted as "
                                            "for the bf16 stack)")
            del x, ws_l, y
    return out


def run_ours(args, world, rank, local):
    import softmax_attention_sana_b200 as sana
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    grid = (WL.T, WL.H, WL.W)
    cpu_inputs = si.qkvg(WL)
    q, k, v, g = (t.to(dev) for t in cpu_inputs)
    rope = sana.Rope(WL.T, WL.H, WL.W, WL.rope_split)
    ws = torch.empty(sana.linattn_workspace_size(WL.B, grid, WL.heads, WL.D, 1), dtype=torch.uint8,
                     device=dev)
    y = torch.empty_like(q)
    step = lambda: sana.linattn_fwd(q, k, v, g, rope, grid, WL.heads, out=y, ws=ws)

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    sana.sync_status()
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark("t0")
    ms_local = time_loop(step, args.steps)
    barrier(world)
    clocks.mark("t1")
    sana.sync_status()
    rate, ms = whole_job_rate(WL.B * WL.N, ms_local, world)
    clk = clocks.stop()

    # dominant kernel: the output pass (Q, G read, Y written), one launch per call
    S, z = sana.linattn_state(k, v, rope, grid, WL.heads)
    apply = lambda: sana.linattn_apply(q, g, rope, grid, WL.heads, S, z, out=y)
    for _ in range(3):
        apply()
    ms_apply = time_loop(apply, max(10, args.steps))
    st_ws = torch.empty(max(256, sana._lib.linattn_state_workspace_size(WL.B, grid, WL.heads, WL.D, 1)),
                        dtype=torch.uint8, device=dev)
    state = lambda: sana.linattn_state(k, v, rope, grid, WL.heads, S=S, z=z, ws=st_ws)
    for _ in range(3):
        state()
    ms_state = time_loop(state, max(10, args.steps))
    sana.sync_status()

    # end to end through the C ABI from pinned host buffers: every step copies
    # its Q, K, V, G in and its Y out; two device buffer sets and three streams
    # let step i's output copy and compute overlap step i+1's input copies
    # (PCIe is full duplex), as a pipeline of layers would run
    hq, hk, hv, hg = (t.cpu().pin_memory() for t in (q, k, v, g))
    hy = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    dbuf = [tuple(torch.empty_like(t) for t in (q, k, v, g)) for _ in range(2)]
    ybuf = [y, torch.empty_like(y)]
    s_in, s_run, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_run + ev_out:
        e.record(torch.cuda.current_stream())

    def e2e_step(i):
        b = i & 1
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_run[b])  # buffer set b is no longer read by step i - 2
            for d, h in zip(dbuf[b], (hq, hk, hv, hg)):
                d.copy_(h, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[b])
            s_run.wait_event(ev_out[b])  # ybuf[b] of step i - 2 has been copied out
            sana.linattn_fwd(*dbuf[b], rope, grid, WL.heads, out=ybuf[b], ws=ws)
            ev_run[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[b])
            hy[b].copy_(ybuf[b], non_blocking=True)
            ev_out[b].record(s_out)

    def e2e_time(steps):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record()
        for st_ in (s_in, s_run, s_out):
            st_.wait_event(t0)
        for i in range(steps):
            e2e_step(i)
        cur = torch.cuda.current_stream()
        for st_ in (s_in, s_run, s_out):
            cur.wait_stream(st_)
        t1.record()
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / steps

    e2e_time(2)
    ms_e2e = max_over_ranks(e2e_time(args.e2e_steps), world)
    sana.sync_status()

    comp = components(sana, args) if (world == 1 and args.components == "all") else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, dt, desc = oracle_sample(args.ref_heads, WL.N, cpu_inputs)
        cpu = {"value": v_cpu, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc + f" ({dt:.1f} s of CPU time)"}

    if rank != 0:
        return
    hbm, peak_kind = peaks()
    ach_apply = APPLY_BYTES / (ms_apply / 1e3) / 1e9
    ach_layer = LAYER_BYTES / (ms / 1e3) / 1e9
    tokens = world * WL.B * WL.N
    line = {
        "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(),
        "tflops_per_layer": LAYER_FLOPS / (ms / 1e3) / 1e12,
        "roofline": {"bound": "hbm", "kernel": "linattn_out_kernel (output pass: Q, G read, Y written)",
                     "achieved": ach_apply, "peak": hbm, "unit": "GB/s", "frac": ach_apply / hbm,
                     "peak_kind": peak_kind, "traffic": recorded_traffic(),
                     "algorithmic_bytes_per_launch": APPLY_BYTES, "ms_per_launch": ms_apply},
        "layer_roofline": {"bound": "hbm", "achieved": ach_layer, "peak": hbm, "unit": "GB/s",
                           "frac": ach_layer / hbm, "algorithmic_bytes": LAYER_BYTES,
                           "state_phase_ms": ms_state, "apply_phase_ms": ms_apply},
        "e2e": {"value": tokens / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": 4 * TENSOR_BYTES, "d2h_bytes_per_step": TENSOR_BYTES,
                "ms_per_step": ms_e2e,
                "pipelining": "two device buffer sets; step i's compute and output copy overlap "
                              "step i+1's input copies"},
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    if comp is not None:
        anchor_roof = comp.pop("_anchor_roofline", None)
        if anchor_roof is not None:
            line["anchor_roofline"] = anchor_roof
        line["components"] = comp
    print(json.dumps(line), flush=True)


def chunk_step_times(steps=64):
    """The 720p/60s block-causal chunk step (3 frames, 10,800 tokens, ungated,
    state carried): device ms per step back to back over 4 distinct chunks,
    ms of one isolated call after an L2 flush, and the bytes of one step."""
    import softmax_attention_sana_b200 as sana
    wl = si.LONG
    grid = (3, wl.H, wl.W)
    chunks = [tuple(t.cuda() for t in si.causal_chunk(wl, i, 3)) for i in range(4)]
    rope = sana.Rope(wl.T, wl.H, wl.W, wl.rope_split)
    S = torch.zeros(1, wl.heads, wl.D, wl.D, device="cuda")
    z = torch.zeros(1, wl.heads, wl.D, device="cuda")
    ws = torch.empty(sana.linattn_workspace_size(1, grid, wl.heads, wl.D, 1), dtype=torch.uint8,
                     device="cuda")
    ys = [torch.empty_like(c[0]) for c in chunks]
    it = [0]

    def f():
        i = it[0] % 4
        q, k, v = chunks[i]
        sana.linattn_block_causal_step(q, k, v, None, rope, grid, 3 * i, wl.heads, S, z,
                                       commit=True, out=ys[i], ws=ws)
        it[0] += 1

    for _ in range(8):
        f()
    ms_b2b = time_loop(f, steps)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tot = 0.0
    for _ in range(20):
        flush.zero_()
        torch.cuda.synchronize()
        s_ev.record()
        f()
        e_ev.record()
        torch.cuda.synchronize()
        tot += s_ev.elapsed_time(e_ev)
    sana.sync_status()
    nb = 4 * 10800 * wl.C * 2 + 2 * 4 * wl.heads * (wl.D * wl.D + wl.D)
    return ms_b2b, tot / 20, nb


def run_chunk_only(args):
    """The 720p/60s block-causal chunk step: ms per step (back to back) and of
    one isolated call."""
    ms_b2b, ms_iso, nb = chunk_step_times(args.steps)
    print(json.dumps({"causal_chunk_720p60s_ms": ms_b2b, "isolated_ms": ms_iso,
                      "GB_per_s": nb / (ms_b2b / 1e3) / 1e9}), flush=True)


def run_anchor_only(args):
    """The softmax anchor on the 480p grid (N = 32,760), or with --anchor-720p
    on the 720p/5s grid (N = 75,600): K steps, ms per call."""
    import softmax_attention_sana_b200 as sana
    wl = si.P720 if args.anchor_720p else si.P480
    q, k, v, g = (t.cuda() for t in si.qkvg(wl))
    rope = sana.Rope(wl.T, wl.H, wl.W, wl.rope_split)
    y = torch.empty_like(q)
    f = lambda: sana.softmax_anchor_fwd(q, k, v, g, rope, (wl.T, wl.H, wl.W), wl.heads, out=y)
    for _ in range(args.warmup):
        f()
    ms = time_loop(f, args.steps)
    sana.sync_status()
    flops = 4 * wl.N * wl.N * wl.heads * wl.D
    name = "anchor_720p_ms" if args.anchor_720p else "anchor_480p_ms"
    print(json.dumps({name: ms, "TFLOP_per_s": flops / (ms / 1e3) / 1e12}), flush=True)


def run_scan_only(args):
    """The whole 720p/60s sequence through the block-causal scan (81 blocks,
    867,600 tokens, inputs drawn on the device): K steps, ms per call."""
    import softmax_attention_sana_b200 as sana
    wl = si.LONG
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4000)
    q, k, v = (torch.randn((1, wl.N, wl.C), generator=gen, device="cuda", dtype=torch.bfloat16)
               for _ in range(3))
    rope = sana.Rope(wl.T, wl.H, wl.W, wl.rope_split)
    S = torch.zeros(1, wl.heads, wl.D, wl.D, device="cuda")
    z = torch.zeros(1, wl.heads, wl.D, device="cuda")
    ws = torch.empty(sana.linattn_block_causal_scan_workspace_size(1, (wl.T, wl.H, wl.W), wl.heads,
                                                                   wl.D, 3, 1),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty_like(q)
    f = lambda: sana.linattn_block_causal_scan(q, k, v, None, rope, (wl.T, wl.H, wl.W), 0,
                                               wl.heads, 3, S, z, commit=False, out=y, ws=ws)
    for _ in range(args.warmup):
        f()
    ms = time_loop(f, args.steps)
    sana.sync_status()
    nb = 4 * wl.N * wl.C * 2 + 2 * wl.heads * (wl.D * wl.D + wl.D) * 4
    print(json.dumps({"scan_720p60s_ms": ms, "tokens_per_s": wl.N / (ms / 1e3),
                      "GB_per_s": nb / (ms / 1e3) / 1e9}), flush=True)


def run_bwd_only(args):
    """Backward of the gated linear-attention layer at 720p/5s (dq, dk, dv, dg
    from dy; S and z recomputed): K steps, ms per call."""
    import softmax_attention_sana_b200 as sana
    q, k, v, g = (t.cuda() for t in si.qkvg(WL))
    dy = si.normal(7000, (1, WL.N, WL.C)).cuda()
    grid = (WL.T, WL.H, WL.W)
    rope = sana.Rope(WL.T, WL.H, WL.W, WL.rope_split)
    f = lambda: sana.linattn_bwd(q, k, v, g, rope, grid, WL.heads, dy)
    for _ in range(args.warmup):
        f()
    ms = time_loop(f, args.steps)
    sana.sync_status()
    nb = 9 * TENSOR_BYTES  # q, k, v, g, dy read once; dq, dk, dv, dg written once
    print(json.dumps({"linattn_bwd_720p_ms": ms, "tokens_per_s": WL.N / (ms / 1e3),
                      "GB_per_s": nb / (ms / 1e3) / 1e9}), flush=True)
    S, z = sana.linattn_state(k, v, rope, grid, WL.heads)
    f = lambda: sana.linattn_bwd(q, k, v, g, rope, grid, WL.heads, dy, S=S, z=z)
    for _ in range(args.warmup):
        f()
    ms = time_loop(f, args.steps)
    sana.sync_status()
    print(json.dumps({"linattn_bwd_saved_state_720p_ms": ms, "tokens_per_s": WL.N / (ms / 1e3),
                      "GB_per_s": nb / (ms / 1e3) / 1e9}), flush=True)
    del q, k, v, g, dy, S, z
    # the AttnRes router's backward over 3 sources: 3 sources and dh read,
    # 3 source gradients written
    srcs = [t.cuda() for t in si.attnres_sources(5, 3, 1, WL.N, WL.C)]
    w_attn, _ = (t.cuda() for t in si.router_queries(5, WL.C))
    dh = si.normal(7100, (1, WL.N, WL.C)).cuda()
    wsb = torch.empty(sana._lib.lib.sana_attnres_route_bwd_workspace_size(1, WL.N, WL.C),
                      dtype=torch.uint8, device="cuda")
    f = lambda: sana.attnres_route_bwd(srcs, w_attn, dh, ws=wsb)
    for _ in range(args.warmup):
        f()
    ms = time_loop(f, args.steps)
    sana.sync_status()
    print(json.dumps({"attnres_route_bwd_720p_3src_ms": ms,
                      "GB_per_s": 7 * TENSOR_BYTES / (ms / 1e3) / 1e9}), flush=True)


def run_sparse_only(args):
    """The block-sparse anchor on the 720p/5s grid, a quarter of the key tiles
    per 256-query block (selection included): K steps, ms per call."""
    import softmax_attention_sana_b200 as sana
    q, k, v, g = (t.cuda() for t in si.qkvg(WL))
    grid = (WL.T, WL.H, WL.W)
    rope = sana.Rope(WL.T, WL.H, WL.W, WL.rope_split)
    nkt = sana.anchor_tile_count(WL.N)
    keep = (nkt + 3) // 4
    y = torch.empty_like(q)
    ws = torch.empty(sana.softmax_anchor_sparse_workspace_size(1, grid, WL.heads, WL.D),
                     dtype=torch.uint8, device="cuda")
    tiles = torch.empty(1, WL.heads, (nkt + 1) // 2, keep, dtype=torch.int32, device="cuda")
    f = lambda: sana.softmax_anchor_sparse_fwd(q, k, v, g, rope, grid, WL.heads, keep, tiles=tiles,
                                               out=y, ws=ws)
    for _ in range(args.warmup):
        f()
    ms = time_loop(f, args.steps)
    sana.sync_status()
    kept = 4 * WL.N * min(WL.N, keep * 128) * WL.heads * WL.D
    print(json.dumps({"sparse_anchor_720p_25pct_ms": ms, "keep_tiles": keep,
                      "TFLOP_per_s_executed": kept / (ms / 1e3) / 1e12}), flush=True)


def run_gemm_only(args):
    """The bf16 QKVG projection GEMM of the 720p stack ((75,600 x 3072) .
    (12,288 x 3072)^T): K steps."""
    import softmax_attention_sana_b200 as sana
    A = torch.randn(WL.N, WL.C, device="cuda", dtype=torch.bfloat16)
    W = torch.randn(4 * WL.C, WL.C, device="cuda", dtype=torch.bfloat16) * WL.C ** -0.5
    Y = torch.empty(WL.N, 4 * WL.C, device="cuda", dtype=torch.bfloat16)
    f = lambda: sana.gemm_bf16(A, W, out=Y)
    for _ in range(args.warmup):
        f()
    ms = time_loop(f, args.steps)
    sana.sync_status()
    flops = 2 * WL.N * 4 * WL.C * WL.C
    print(json.dumps({"gemm_qkvg_720p_ms": ms, "TFLOP_per_s": flops / (ms / 1e3) / 1e12}),
          flush=True)


def run_mx_only(args):
    """The MX projection of the 720p QKVG shape (75,600 x 3072 activations
    quantised on the fly against 12,288 x 3072 MXFP4 weights): K steps."""
    import softmax_attention_sana_b200 as sana
    A = torch.randn(WL.N, WL.C, device="cuda", dtype=torch.bfloat16)
    W = torch.randn(4 * WL.C, WL.C, device="cuda", dtype=torch.bfloat16) * WL.C ** -0.5
    Y = torch.empty(WL.N, 4 * WL.C, device="cuda", dtype=torch.bfloat16)
    wq, wsc = sana.mx_quantize(W, fp4=True)
    ws = torch.empty(sana._lib.lib.sana_mx_linear_workspace_size(WL.N, WL.C), dtype=torch.uint8,
                     device="cuda")
    f = lambda: sana.mx_linear(A, wq, wsc, 4 * WL.C, out=Y, ws=ws)
    for _ in range(args.warmup):
        f()
    ms = time_loop(f, args.steps)
    sana.sync_status()
    flops = 2 * WL.N * 4 * WL.C * WL.C
    print(json.dumps({"mx_linear_qkvg_720p_ms": ms, "TFLOP_per_s": flops / (ms / 1e3) / 1e12}),
          flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--components", choices=["all", "none"], default="all")
    ap.add_argument("--ref-heads", type=int, default=12,
                    help="heads of the 720p layer in the cpu_baseline sample")
    ap.add_argument("--ref-budget", type=float, default=150.0,
                    help="seconds the --impl reference run aims to take")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-anchor", action="store_true", help="leave the anchor out of the components")
    ap.add_argument("--no-stacks", action="store_true",
                    help="leave the 4-layer group and the 16-layer AttnRes stack out of the components")
    ap.add_argument("--anchor-only", action="store_true",
                    help="run only the 480p-shaped softmax anchor (a small case for profiling)")
    ap.add_argument("--scan-only", action="store_true",
                    help="run only the whole-sequence block-causal scan at 720p/60s")
    ap.add_argument("--bwd-only", action="store_true",
                    help="run only the linear-attention backward at 720p/5s")
    ap.add_argument("--sparse-only", action="store_true",
                    help="run only the block-sparse anchor at 720p/5s (25%% of the key tiles)")
    ap.add_argument("--anchor-720p", action="store_true",
                    help="with --anchor-only: the 720p/5s grid instead of 480p")
    ap.add_argument("--gemm-only", action="store_true",
                    help="only the bf16 QKVG projection GEMM at 720p")
    ap.add_argument("--mx-only", action="store_true",
                    help="run only the MX projection of the 720p QKVG shape")
    ap.add_argument("--chunk-only", action="store_true",
                    help="run only the 720p/60s block-causal chunk step (K steps back to back)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup() if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.anchor_only:
            run_anchor_only(args)
            return
        if args.scan_only:
            run_scan_only(args)
            return
        if args.sparse_only:
            run_sparse_only(args)
            return
        if args.bwd_only:
            run_bwd_only(args)
            return
        if args.chunk_only:
            run_chunk_only(args)
            return
        if args.mx_only:
            run_mx_only(args)
            return
        if args.gemm_only:
            run_gemm_only(args)
            return
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
