#!/usr/bin/env python
"""Benchmark of the Flint MoE layer decode step on B200 (one JSON line on stdout).

Default workload: the Flint-shaped layer (d=2048, I=512, 256 routed + 1 shared
experts, top-6, NVFP4 W4A16) at decode batch 1. A step is one layer call: router
GEMV, softmax/top-6, grouping, gate/up and down dequant-GEMVs, gated combine.
To keep weights out of L2, 47 independently drawn layers (21.4 GB of packed
weights, resident in HBM) are used in turn, each step's output (plus its input
as the residual) feeding the next step, as in decode through the 47-layer stack.
Steps are replayed from a CUDA graph of PDL-chained layer calls.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl flint|reference]

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only). With N > 1 each rank runs an independent replica on its
own GPU (the layer has no exchange step); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer decode tokens/s at batch 1 (achieved HBM GB/s vs ~8 TB/s reported alongside)"
UNIT = "tokens/s"
N_LAYERS = 47
NOMINAL_HBM_GBS = 8000.0


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _tensor_peak(wdtype: str):
    """Dense tensor peak (TFLOP/s) of the MMA's operand type: the measured bf16
    figure (f16 runs at the same rate on tcgen05 kind::f16)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), "measured (bf16 burst; f16 operands run at the bf16 rate)"
    except Exception:
        return 1590.0, "fallback"


# DRAM bytes (read + write) of one launch of the batch-1 cluster kernel
# (k_tok1<2048, 512>), from an ncu capture of `bench.py --profile t1`
# (13,482,752 read + 0 written: the seven experts, the router rows and x);
# None whenever the kernel changes until it is captured again.
TRAFFIC_K_TOK1 = 13482752


def _host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ----------------------------------------------------------------------------- flint arm
class Stack:
    """`n` independently drawn layers of one shape, packed NVFP4 (or laid out in
    bf16), resident on the GPU."""

    def __init__(self, w: synth.Workload, n: int, seed: int, max_tokens: int, wdtype: str = "nvfp4"):
        import torch
        import nvfp4_weight_only_flint_b200 as fm
        self.fm, self.w, self.wdtype = fm, w, wdtype
        self.shape = fm.Shape(w.d, w.inter, w.E, w.k, w.S, fm.FLINT_W_NVFP4 if wdtype == "nvfp4" else fm.FLINT_W_BF16)
        self.ws = torch.empty(fm.flint_moe_workspace_bytes(self.shape, max_tokens), dtype=torch.uint8, device="cuda")
        fm.flint_moe_workspace_init(self.ws)
        self.layers = []
        for l in range(n):
            wf = synth.layer_weights_torch(seed, l, w.E + w.S, w.d, w.inter, w.std, device="cuda")
            if wdtype == "nvfp4":
                packed = torch.empty(fm.flint_packed_bytes(self.shape), dtype=torch.uint8, device="cuda")
                scales = torch.empty(fm.flint_block_scale_bytes(self.shape), dtype=torch.uint8, device="cuda")
                ts = torch.empty((w.E + w.S) * 3, dtype=torch.float32, device="cuda")
                fm.flint_pack_nvfp4(wf, 0, self.shape, packed, scales, ts, self.ws)
                wts = fm.Weights(packed.data_ptr(), scales.data_ptr(), ts.data_ptr())
            else:
                wb = wf.to(torch.bfloat16)
                packed = torch.empty(fm.flint_packed_bytes(self.shape) // 2, dtype=torch.int16, device="cuda")
                fm.flint_pack_bf16(wb.view(torch.int16), self.shape, packed)
                torch.cuda.synchronize()
                del wb
                scales = ts = None
                wts = fm.Weights(packed.data_ptr(), None, None)
            del wf
            self.layers.append((packed, scales, ts, wts))
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    def expert_bytes(self):
        """(gate+up, down) bytes of one expert: codes and block scales, or bf16."""
        w = self.w
        if self.wdtype == "bf16":
            return 2 * w.inter * w.d * 2, w.inter * w.d * 2
        gu = w.inter * w.d // 2 * 2 + w.inter * w.d // 16 * 2
        dn = w.inter * w.d // 2 + w.inter * w.d // 16
        return gu, dn


def _bits_to_cuda(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def run_chain(stack: Stack, routers, T: int, K: int, W: int, sampler=None, residual=True,
              fixed_inputs=None, norm: int = 0, variant: int = 0):
    """Time exactly K layer steps replayed from CUDA graphs. With fixed_inputs
    (one x per layer) steps are independent; otherwise each step's output is
    the next step's input (residual chain)."""
    import torch
    fm = stack.fm
    L = len(stack.layers)
    d = stack.w.d
    stream = torch.cuda.Stream()
    bufs = [torch.zeros((T, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    x0 = _bits_to_cuda(synth.x_bits(12345, T, d))
    bufs[0].copy_(x0)
    opt = fm.Options(path=fm.FLINT_PATH_AUTO, use_pdl=1, input_rmsnorm=norm, layer_variant=variant)
    P = 2 * L

    def step(s):
        l = s % L
        if fixed_inputs is not None:
            xin, out, res = fixed_inputs[l], bufs[s % 2], None
        else:
            xin, out = bufs[s % 2], bufs[(s + 1) % 2]
            res = xin if residual else None
        fm.flint_moe_forward_ex(xin, T, routers[l], stack.layers[l][3], stack.shape, res, out, stack.ws, opt)

    with torch.cuda.stream(stream):
        for s in range(P):  # eager warm-up (sets kernel attributes before capture)
            step(s)
    torch.cuda.synchronize()

    def capture(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for s in range(n):
                step(s)
        return g

    # the timed region replays g_full K // P times and g_rem once; every graph
    # it replays is replayed (untimed) first, at least W steps in all
    n_full, rem = K // P, K % P
    g_full = capture(P) if n_full else None
    g_rem = capture(rem) if rem else None
    with torch.cuda.stream(stream):
        done = 0
        while True:
            if g_full is not None:
                g_full.replay()
                done += P
            if g_rem is not None:
                g_rem.replay()
                done += rem
            if done >= W:
                break
    torch.cuda.synchronize()
    if fixed_inputs is None:
        bufs[0].copy_(x0)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(n_full):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()
        end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    _barrier()
    ms = start.elapsed_time(end)
    rc, flags = fm.flint_moe_get_status(stack.ws)
    if rc != 0:
        raise RuntimeError(f"device status {rc} flags {flags}")
    del g_full, g_rem
    return ms, clocks


def kernel_timing(stack: Stack, routers, T: int, n_calls: int, fixed_inputs=None, norm: int = 0):
    """Per-launch duration of the kernel that streams the expert weights (CUDA
    events the library records on the launching stream around it: the
    persistent layer kernel at T <= 8, the gate/up tensor-core kernel from 32)
    and its algorithmic bytes and flops per launch."""
    import torch
    fm = stack.fm
    L = len(stack.layers)
    w = stack.w
    gu, dn = stack.expert_bytes()
    stream = torch.cuda.Stream()
    x = _bits_to_cuda(synth.x_bits(777, T, w.d))
    out = torch.empty_like(x)
    ids = torch.empty((n_calls, T, w.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((n_calls, T, w.k), dtype=torch.float32, device="cuda")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_calls)]
    handles = []
    for e0, e1 in evs:
        e0.record(stream)  # materialise the CUDA events
        e1.record(stream)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(n_calls):
            l = i % L
            xin = fixed_inputs[l] if fixed_inputs is not None else x
            arr = (ctypes_void_p * 2)(evs[i][0].cuda_event, evs[i][1].cuda_event)
            handles.append(arr)
            opt = fm.Options(path=fm.FLINT_PATH_AUTO, use_pdl=1, topk_ids=ids[i].data_ptr(),
                             topk_weights=gates[i].data_ptr(), input_rmsnorm=norm,
                             profile_events=ctypes_addressof(arr))
            fm.flint_moe_forward_ex(xin, T, routers[l], stack.layers[l][3], stack.shape, None, out, stack.ws, opt)
    torch.cuda.synchronize()
    ms = [evs[i][0].elapsed_time(evs[i][1]) for i in range(n_calls)]
    ids_np = ids.cpu().numpy()
    byt, flops = [], []
    P = T * (w.k + w.S)
    for i in range(n_calls):
        U = len(np.unique(ids_np[i]))
        if T <= 8:
            # the whole layer: union of the selected experts + the shared one, x in, out
            byt.append(step_bytes(w, ids_np[i], stack.wdtype))
            flops.append(2.0 * P * 3 * w.inter * w.d)
        else:
            # gate/up on the tensor cores: the union's gate/up weights, the
            # gathered activation rows (16-bit) in, h (fp32) out
            byt.append((U + w.S) * gu + P * w.d * 2 + P * w.inter * 4)
            flops.append(2.0 * P * 2 * w.inter * w.d)
    skip = min(n_calls // 4, L)  # first launches warm the code paths
    return float(np.mean(ms[skip:])), float(np.mean(byt[skip:])), float(np.mean(flops[skip:])), ids_np


def step_bytes(w: synth.Workload, ids_np, wdtype: str = "nvfp4"):
    """Byte count of one step: union of the selected experts' weights and
    scales plus the shared expert's, plus x in and out (bf16)."""
    if wdtype == "bf16":
        per = 3 * w.inter * w.d * 2
    else:
        per = 3 * (w.inter * w.d // 2 + w.inter * w.d // 16)
    U = len(np.unique(ids_np))
    return (U + w.S) * per + 2 * ids_np.shape[0] * w.d * 2


def run_e2e(stack: Stack, routers, T: int, K: int, norm: int = 0):
    """The same metric through the public call with host buffers: each step
    copies x (pinned host) to the device, runs the layer and copies out back."""
    import torch
    fm = stack.fm
    L = len(stack.layers)
    d = stack.w.d
    stream = torch.cuda.Stream()
    xs_host = [torch.from_numpy(synth.x_bits(900 + i, T, d).view(np.int16)).view(torch.bfloat16).pin_memory()
               for i in range(8)]
    out_host = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    out_dev = torch.empty_like(x_dev)
    opt = fm.Options(path=fm.FLINT_PATH_AUTO, use_pdl=1, input_rmsnorm=norm)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for i in range(2 * L):
            x_dev.copy_(xs_host[i % 8], non_blocking=True)
            fm.flint_moe_forward_ex(x_dev, T, routers[i % L], stack.layers[i % L][3], stack.shape, None, out_dev,
                                    stack.ws, opt)
            out_host.copy_(out_dev, non_blocking=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(K):
            x_dev.copy_(xs_host[i % 8], non_blocking=True)
            fm.flint_moe_forward_ex(x_dev, T, routers[i % L], stack.layers[i % L][3], stack.shape, None, out_dev,
                                    stack.ws, opt)
            out_host.copy_(out_dev, non_blocking=True)
        end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    return T * K / (ms / 1e3), T * d * 2, T * d * 2


LM_VOCAB = 150144


def run_lm_head(world: int, n_heads: int = 3, calls: int = 60):
    """The 4-bit output head (150,144 x 2048 NVFP4, 173 MB): a graph of `calls`
    launches cycling through `n_heads` independently drawn heads (more than
    L2 holds), per launch time from CUDA events on the launching stream."""
    import torch
    import nvfp4_weight_only_flint_b200 as fm
    rows, cols = LM_VOCAB, 2048
    ws = torch.zeros(2048, dtype=torch.uint8, device="cuda")
    heads = []
    for h in range(n_heads):
        gen = torch.Generator(device="cuda")
        gen.manual_seed(synth.key(0, "experts", 10000 + h) & 0x7FFFFFFFFFFFFFFF)
        w = torch.randn((rows, cols), generator=gen, device="cuda", dtype=torch.float32).mul_(0.02)
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
        scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device="cuda")
        ts = torch.empty(4, dtype=torch.float32, device="cuda")
        fm.flint_pack_nvfp4_dense(w, 0, rows, cols, codes, scales, ts, ws)
        torch.cuda.synchronize()
        del w
        heads.append((codes, scales, ts))
    peak, peak_kind = _peaks()
    res = {"workload": f"dense NVFP4 output head {rows} x {cols} (173 MB), {n_heads} heads used in turn",
           "kernel": "k_lm_head"}
    st = torch.cuda.Stream()
    for T in (1, 8):
        x = _bits_to_cuda(synth.x_bits(4242, T, cols))
        out = torch.empty((T, rows), dtype=torch.float32, device="cuda")
        with torch.cuda.stream(st):
            for i in range(2 * n_heads):
                c, s_, t_ = heads[i % n_heads]
                fm.flint_lm_head(x, T, c, s_, t_, rows, cols, out, ws)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            for i in range(calls):
                c, s_, t_ = heads[i % n_heads]
                fm.flint_lm_head(x, T, c, s_, t_, rows, cols, out, ws)
        with torch.cuda.stream(st):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(st):
            e0.record(st)
            g.replay()
            e1.record(st)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / calls * 1e3
        byt = rows * cols // 2 + rows * cols // 16 + T * cols * 2 + T * rows * 4
        res[f"batch{T}"] = {"us": us, "bytes": byt, "gbs": byt / us / 1e3, "frac_of_peak": byt / us / 1e3 / peak,
                            "tokens_per_s": world * T / (us / 1e6)}
        del g
    rc, flags = fm.flint_moe_get_status(ws)
    if rc != 0:
        raise RuntimeError(f"lm head status {rc} flags {flags}")
    del heads
    torch.cuda.empty_cache()
    return res


def run_prefill(world: int, seed: int, T: int = 8192, n_layers: int = 4, calls: int = 12):
    """One prefill-size call of 8192 tokens per layer on the tensor-core path
    (counting-sort grouping, 128-token tiles), NVFP4 weights of the Flint
    shape, 4 resident layers used in turn; the expert GEMMs' rate against the
    16-bit tensor peak (the operands are f16, e2m1*e4m3 exact)."""
    import torch
    w = synth.CONFIGS["cfg1"]
    st = Stack(w, n_layers, seed, max_tokens=T)
    xs = [_bits_to_cuda(synth.x_bits(seed + 3000 + l, T, w.d)) for l in range(n_layers)]
    rs = [_bits_to_cuda(synth.to_bf16_bits(synth.router_plain(seed, w.d, w.E, l))) for l in range(n_layers)]
    ms, _ = run_chain(st, rs, T, calls, n_layers, fixed_inputs=xs)
    ms = _max_over_ranks(ms)
    per = ms / calls / 1e3
    P = T * (w.k + w.S)
    flops = 2.0 * P * 3 * w.inter * w.d
    tf_peak, tf_kind = _tensor_peak("nvfp4")
    del st, xs
    torch.cuda.empty_cache()
    return {"workload": f"{T} tokens through one d=2048/I=512/E=256+1 top-6 NVFP4 layer (prefill-size call)",
            "ms_per_layer": per * 1e3, "tokens_per_s": world * T / per,
            "expert_tflops": flops / per / 1e12, "frac_of_tensor_peak": flops / per / 1e12 / tf_peak,
            "tensor_peak_tflops": tf_peak, "tensor_peak_kind": tf_kind}


def run_attn_prologue(seed: int, calls: int = 50):
    """The attention prologue (flint_qk_norm_rope_kv) at the pages' heads (32
    query, 4 key/value, dimension 128), rotary on: per-call device time from a
    CUDA graph of `calls` launches, at decode and prefill sizes, with the
    bytes it must move (qkv in, cos/sin row, q out, k and v into the cache)."""
    import torch
    import nvfp4_weight_only_flint_b200 as fm
    hq, hkv, dh = 32, 4, 128
    res = {"workload": "fused Q/K RMS norm + rotary + KV-cache write, 32 q / 4 kv heads x 128, bf16"}
    peak, kind = _peaks()
    for T in (1, 64, 8192):
        g = torch.Generator(device="cuda").manual_seed(seed + T)
        qkv = torch.randn((T, hq + 2 * hkv, dh), device="cuda", generator=g).to(torch.bfloat16)
        w = torch.ones(dh, device="cuda").to(torch.bfloat16)
        max_pos = max(T, 4096)
        inv = 10000.0 ** (-torch.arange(0, dh, 2, device="cuda", dtype=torch.float64) / dh)
        ang = torch.arange(max_pos, device="cuda", dtype=torch.float64)[:, None] * inv[None, :]
        cs = torch.cat([ang.cos(), ang.sin()], dim=1).float().contiguous()
        pos = torch.arange(T, device="cuda", dtype=torch.int32)
        slots = torch.arange(T, device="cuda", dtype=torch.int32)
        q_out = torch.empty((T, hq, dh), device="cuda", dtype=torch.bfloat16)
        kc = torch.empty((T, hkv, dh), device="cuda", dtype=torch.bfloat16)
        vc = torch.empty((T, hkv, dh), device="cuda", dtype=torch.bfloat16)
        st = torch.cuda.Stream()

        def call():
            fm.flint_qk_norm_rope_kv(qkv, T, hq, hkv, w, w, cs, max_pos, pos, True, 1e-6, slots, T, q_out, kc, vc,
                                     stream=st.cuda_stream)
        with torch.cuda.stream(st):
            for _ in range(5):
                call()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=st):
            for _ in range(calls):
                call()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(st):  # replay and events on the captured stream
            graph.replay()
            torch.cuda.synchronize()
            e0.record()
            graph.replay()
            e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / calls * 1e3
        byt = T * ((hq + 2 * hkv) * dh * 2 + dh * 4 + (hq + 2 * hkv) * dh * 2 + 8)
        res[f"T{T}"] = {"us": us, "bytes": byt, "gbs": byt / (us * 1e-6) / 1e9, "frac_of_peak": byt / (us * 1e-6) / 1e9 / peak}
        del graph
    return res


def run_decode_attention(seed: int, calls: int = 40):
    """Decode attention (flint_decode_attention) at the pages' heads (32 query,
    4 key/value, dimension 128) over bf16 caches: per-call device time from a
    CUDA graph of `calls` launches, the calls cycling over cache regions of
    more than 300 MB in all so that no call finds its rows in L2; bytes = the
    key and value rows read (2 KB per row and token) plus q and out."""
    import torch
    import nvfp4_weight_only_flint_b200 as fm
    hq, hkv, dh = 32, 4, 128
    res = {"workload": "GQA decode attention, 32 q / 4 kv heads x 128, bf16 cache, split-K over the context"}
    peak, kind = _peaks()
    row_bytes = hkv * dh * 2 * 2
    for T, L in ((1, 4096), (1, 32768), (1, 131072), (8, 32768), (64, 4096)):
        regions = max(1, -(-(300 << 20) // (T * L * row_bytes)))
        rows = regions * T * L
        g = torch.Generator(device="cuda").manual_seed(seed + T * 7 + L)
        kc = torch.randn((rows, hkv, dh), device="cuda", generator=g).to(torch.bfloat16)
        vc = torch.randn((rows, hkv, dh), device="cuda", generator=g).to(torch.bfloat16)
        q = torch.randn((T, hq, dh), device="cuda", generator=g).to(torch.bfloat16)
        out = torch.empty((T, hq, dh), device="cuda", dtype=torch.bfloat16)
        length = torch.full((T,), L, device="cuda", dtype=torch.int32)
        starts = [torch.arange(T, device="cuda", dtype=torch.int64) * L + r * T * L for r in range(regions)]
        nb = fm.flint_decode_attention_workspace_bytes(T, hkv, L)
        ws = torch.empty(max(nb, 16), device="cuda", dtype=torch.uint8) if nb else None
        st = torch.cuda.Stream()

        def call(i):
            fm.flint_decode_attention(q, kc, vc, rows, starts[i % regions], length, T, hq, hkv, L, dh ** -0.5, out,
                                      ws, stream=st.cuda_stream)
        with torch.cuda.stream(st):
            for i in range(5):
                call(i)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=st):
            for i in range(calls):
                call(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(st):
            graph.replay()
            torch.cuda.synchronize()
            e0.record()
            graph.replay()
            e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / calls * 1e3
        byt = T * L * row_bytes + 2 * T * hq * dh * 2
        res[f"T{T}_L{L}"] = {"us": us, "bytes": byt, "gbs": byt / (us * 1e-6) / 1e9,
                             "frac_of_peak": byt / (us * 1e-6) / 1e9 / peak}
        del graph, kc, vc
    res["peak_kind"] = kind
    return res


def run_ep(seed: int, R: int = 8, T: int = 64, reps: int = 20):
    """Expert-parallel layer step (config 1's layer, NVFP4, T tokens per rank),
    R ranks emulated on one GPU: every rank's weights (E/R routed experts +
    the shared one) resident, each phase run for every rank in turn, the
    all-to-all replaced by copies between the ranks' buffers (not timed: on a
    node it is NCCL over NVLink). Timed per rank and call with CUDA events:
    route + dispatch, the routed expert call over the received rows, the
    combine (each phase a CUDA graph of all ranks' calls). Reported beside
    them: the bytes a rank sends and receives over NVLink per step and their
    time at the measured 770 GB/s per direction."""
    import torch
    import nvfp4_weight_only_flint_b200 as fm
    from nvfp4_weight_only_flint_b200 import ep
    w = synth.CONFIGS["cfg1"]
    shape = fm.Shape(w.d, w.inter, w.E, w.k, w.S, fm.FLINT_W_NVFP4)
    pshape = ep.packing_shape(shape, R)
    wr = _bits_to_cuda(synth.to_bf16_bits(synth.router_plain(seed, w.d, w.E, 0)))
    full = synth.layer_weights_torch(seed, 0, w.E + w.S, w.d, w.inter, w.std, device="cuda")
    pack_ws = torch.empty(fm.flint_moe_workspace_bytes(pshape, 1), dtype=torch.uint8, device="cuda")
    fm.flint_moe_workspace_init(pack_ws)
    layers, keep = [], []
    for r in range(R):
        wl = ep.slice_rank_weights(full, shape, r, R)
        packed = torch.empty(fm.flint_packed_bytes(pshape), dtype=torch.uint8, device="cuda")
        scales = torch.empty(fm.flint_block_scale_bytes(pshape), dtype=torch.uint8, device="cuda")
        tsc = torch.empty((pshape.n_experts + pshape.n_shared) * 3, dtype=torch.float32, device="cuda")
        fm.flint_pack_nvfp4(wl, 0, pshape, packed, scales, tsc, pack_ws)
        keep.append((packed, scales, tsc))
        layers.append(ep.ExpertParallelLayer(shape, r, R, fm.Weights(packed.data_ptr(), scales.data_ptr(),
                                                                        tsc.data_ptr()), wr, max_tokens=T))
        del wl
    del full
    torch.cuda.synchronize()
    xs = [_bits_to_cuda(synth.x_bits(seed + 900 + r, T, w.d)) for r in range(R)]
    outs = [torch.empty_like(x) for x in xs]
    # one step with the loopback exchange, so every buffer holds real rows
    sc = [l.send(x, T).cpu().tolist() for l, x in zip(layers, xs)]
    n_recv = []
    for dst in range(R):
        n = 0
        for src in range(R):
            off, c = sum(sc[src][:dst]), sc[src][dst]
            layers[dst].recv_x[n:n + c].copy_(layers[src].send_x[off:off + c])
            layers[dst].recv_ids[n:n + c].copy_(layers[src].send_ids[off:off + c])
            layers[dst].recv_gates[n:n + c].copy_(layers[src].send_gates[off:off + c])
            n += c
        n_recv.append(n)
        layers[dst].experts(n)
    for src in range(R):
        n = 0
        for dst in range(R):
            c, at = sc[src][dst], sum(sc[s2][dst] for s2 in range(src))
            layers[src].y_back[n:n + c].copy_(layers[dst].y[at:at + c])
            n += c
        layers[src].finish(T, outs[src])
    torch.cuda.synchronize()
    for l in layers:
        if int(l.status.item()) != 0:
            raise RuntimeError("expert-parallel step: device check flags")

    st = torch.cuda.Stream()

    def timed(fn):
        """Device time per rank and call: a CUDA graph of reps x R calls."""
        with torch.cuda.stream(st):
            for _ in range(3):
                for r in range(R):
                    fn(r)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=st):
            for _ in range(reps):
                for r in range(R):
                    fn(r)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(st):
            graph.replay()
            torch.cuda.synchronize()
            e0.record()
            graph.replay()
            e1.record()
        torch.cuda.synchronize()
        del graph
        return e0.elapsed_time(e1) / (reps * R) * 1e3
    us_send = timed(lambda r: layers[r].send(xs[r], T))
    us_exp = timed(lambda r: layers[r].experts(n_recv[r]))
    us_fin = timed(lambda r: layers[r].finish(T, outs[r]))
    row = w.d * 2
    remote_out = [sum(c for dst, c in enumerate(sc[r]) if dst != r) for r in range(R)]
    remote_in = [sum(sc[src][r] for src in range(R) if src != r) for r in range(R)]
    # out: rows + ids + gates there, rows back; the larger direction sets the time
    b_out = max(remote_out[r] * (row + 8) + remote_in[r] * row for r in range(R))
    b_in = max(remote_in[r] * (row + 8) + remote_out[r] * row for r in range(R))
    link = 770.0
    return {"workload": f"cfg1 layer, NVFP4, {T} tokens per rank, {R} ranks emulated on one GPU "
                        "(E/R = 32 routed + the shared expert per rank)",
            "us_route_dispatch": us_send, "us_expert_call": us_exp, "us_combine": us_fin,
            "rows_received_mean": float(np.mean(n_recv)), "rows_received_max": int(max(n_recv)),
            "nvlink_bytes_per_rank_max": int(max(b_out, b_in)),
            "us_exchange_at_770GBs": max(b_out, b_in) / (link * 1e3),
            "note": "the all-to-all itself is not measured: one GPU per run"}


def cpu_baseline(n_tokens: int = 3, seed: int = 0):
    """The fp64 oracle as it stands, on host cores: T=1 layer decodes of the
    default workload (quantisation of the needed experts is untimed set-up),
    each timed with all host threads offered and with one thread. The oracle
    spreads a call over its expert jobs (k + S = 7 at T = 1), so at most 7
    threads are busy; `cores` reports that number, not the host's."""
    import oracle
    w = synth.CONFIGS["cfg1"]
    host = _host_cores()
    jobs = w.k + w.S
    busy = min(host, jobs)
    t_all, t_one = [], []
    for i in range(n_tokens):
        x = synth.x_bits(seed + 50 + i, 1, w.d)
        wr = synth.make_router(w, seed, x, layer=i)
        ids, _, _ = oracle.topk(oracle.router_logits(x, wr), w.k)
        experts = [None] * (w.E + w.S)
        for e in list(ids[0]) + list(range(w.E, w.E + w.S)):
            g, u, dn = synth.expert_weights_np(seed, i, int(e), w.d, w.inter, w.std)
            experts[int(e)] = (oracle.quantize(g), oracle.quantize(u), oracle.quantize(dn))
        for n_thr, acc in ((host, t_all), (1, t_one)):
            t0 = time.perf_counter()
            oracle.moe_forward(x, wr, experts, d=w.d, inter=w.inter, E=w.E, k=w.k, S=w.S, n_threads=n_thr)
            acc.append(time.perf_counter() - t0)
    per_tok = statistics.median(t_all)
    return {"value": 1.0 / per_tok, "unit": UNIT, "cores": busy, "kind": "oracle",
            "single_thread_value": 1.0 / statistics.median(t_one), "host_threads": host,
            "sample": f"{n_tokens} single-token decodes of the d=2048/I=512/E=256+1 layer (router, top-6, "
                      f"7 SwiGLU experts, combine) in fp64, each timed with {host} threads offered ({busy} busy: one "
                      f"per expert job) and with 1 thread; medians of {n_tokens}; expert quantisation untimed"}


# ----------------------------------------------------------------------------- dist helpers
_DIST = {"on": False}


def _barrier():
    if _DIST["on"]:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(v: float) -> float:
    """The largest v over the ranks (a device time: the job is as slow as its
    slowest rank). NCCL reduces a device tensor, gloo a host one."""
    if not _DIST["on"]:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: float, world: int, steps: int, max_ms: float) -> float:
    """Units all ranks processed per second, over the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=47 * 2 * 200)
    ap.add_argument("--warmup", type=int, default=47 * 2 * 3)
    ap.add_argument("--impl", choices=["flint", "reference"], default="flint")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-extras", action="store_true", help="skip the batch-8 / batch-4 / batch-64 lines")
    ap.add_argument("--profile", choices=["t1", "t8", "t64_nvfp4", "t64_bf16", "prefill", "attn"], default=None,
                    help="profiling case: one layer, --steps eager layer calls, no timing output")
    args = ap.parse_args()
    if args.profile:
        return run_profile_case(args)
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, world)

    import torch
    torch.cuda.set_device(local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
        _DIST["on"] = True

    import nvfp4_weight_only_flint_b200 as fm
    fm.lib()
    w1 = synth.CONFIGS["cfg1"]
    stack = Stack(w1, N_LAYERS, args.seed, max_tokens=8)
    routers1 = [_bits_to_cuda(synth.to_bf16_bits(synth.router_plain(args.seed, w1.d, w1.E, l)))
                for l in range(N_LAYERS)]

    sampler = ClockSampler(local_rank)
    ms, clocks = run_chain(stack, routers1, 1, args.steps, args.warmup, sampler=sampler, norm=1)
    ms = _max_over_ranks(ms)
    K = args.steps
    tok_s = whole_job_rate(1, world, K, ms)
    ms_step = ms / K

    # Each step is exactly one launch of the batch-1 cluster kernel (no other
    # kernel runs in the step), so the timed region gives that kernel's mean
    # launch-to-launch duration inside the graph. One token always selects k
    # distinct experts: the step's bytes are (k + S) experts plus x and out.
    peak, peak_kind = _peaks()
    sb = float(step_bytes(w1, np.arange(w1.k).reshape(1, w1.k)))
    step_gbs = sb / (ms_step / 1e3) / 1e9

    e2e_val, h2d, d2h = run_e2e(stack, routers1, 1, min(K, 4 * N_LAYERS * 10), norm=1)
    e2e_val = _max_over_ranks(-e2e_val) * -1 if world > 1 else e2e_val

    extras = {}
    if not args.no_extras:
        # batch 8 with ~40% overlapping selections: independent steps over the 47 layers
        w2 = synth.CONFIGS["cfg2"]
        xs8 = [synth.x_bits(args.seed + 1000 + l, w2.T, w2.d) for l in range(N_LAYERS)]
        r8 = [_bits_to_cuda(synth.make_router(w2, args.seed, xs8[l], layer=l)) for l in range(N_LAYERS)]
        fx8 = [_bits_to_cuda(x) for x in xs8]
        K8 = 2 * N_LAYERS * 40
        ms8, _ = run_chain(stack, r8, w2.T, K8, 2 * N_LAYERS, fixed_inputs=fx8)
        ms8 = _max_over_ranks(ms8)
        # the same steps through the batch-2..8 cluster kernel (layer_variant CLUSTER)
        ms8c, _ = run_chain(stack, r8, w2.T, K8, 2 * N_LAYERS, fixed_inputs=fx8, variant=stack.fm.FLINT_LAYER_CLUSTER)
        ms8c = _max_over_ranks(ms8c)
        g8_ms, g8_bytes, _, ids8 = kernel_timing(stack, r8, w2.T, 2 * N_LAYERS, fixed_inputs=fx8)
        sb8 = np.mean([step_bytes(w2, ids8[i]) for i in range(ids8.shape[0])])
        unions = [len(np.unique(ids8[i])) for i in range(ids8.shape[0])]
        ov = [synth.overlap_fraction(ids8[i]) for i in range(ids8.shape[0])]
        extras["batch8"] = {"workload": "cfg2: same layer shape, 8 tokens, ~40% of each token's experts shared "
                                        "with another token; independent steps over the 47 resident layers; "
                                        "single kernel with register-fragment tensor-core (mma.sync) inner loops",
                            "tokens_per_s": world * w2.T * K8 / (ms8 / 1e3), "us_per_layer": ms8 / K8 * 1e3,
                            "step_bytes": sb8, "achieved_gbs": sb8 / (ms8 / K8 / 1e3) / 1e9,
                            "frac_of_8tbs": sb8 / (ms8 / K8 / 1e3) / 1e9 / NOMINAL_HBM_GBS,
                            "frac_of_peak": sb8 / (ms8 / K8 / 1e3) / 1e9 / peak,
                            "union_experts_mean": float(np.mean(unions)), "overlap_mean": float(np.mean(ov)),
                            "layer_kernel": {"name": "k_layer (tensor-core variant)", "us": g8_ms * 1e3, "bytes": g8_bytes,
                                             "gbs": g8_bytes / (g8_ms / 1e3) / 1e9,
                                             "frac_of_peak": g8_bytes / (g8_ms / 1e3) / 1e9 / peak},
                            "cluster_kernel": {"name": "k_tokn (layer_variant CLUSTER, not the default)",
                                               "us_per_layer": ms8c / K8 * 1e3,
                                               "frac_of_peak": sb8 / (ms8c / K8 / 1e3) / 1e9 / peak}}
        # 47-layer stack at batch 4 (residual chain)
        w4 = synth.CONFIGS["cfg3_t4"]
        K4 = 2 * N_LAYERS * 40
        ms4, _ = run_chain(stack, routers1, w4.T, K4, 2 * N_LAYERS, norm=1)
        ms4 = _max_over_ranks(ms4)
        # bytes of a batch-4 step: the mean union over one call per layer (the
        # chain's own inputs change every step; the union statistics do not)
        _, b4_bytes, _, _ = kernel_timing(stack, routers1, w4.T, 2 * N_LAYERS, norm=1)
        # batch 64 on the tensor cores (config 4: Zipf-skewed routing), NVFP4
        # and bf16 weights; 8 resident layers used in turn (inputs > L2)
        w4n = synth.CONFIGS["cfg4_nvfp4"]
        extras["batch64"] = {}
        del stack
        torch.cuda.empty_cache()
        for wd in ("nvfp4", "bf16"):
            st64 = Stack(w4n, 8, args.seed, max_tokens=64, wdtype=wd)
            xs64 = [synth.x_bits(args.seed + 2000 + l, w4n.T, w4n.d) for l in range(8)]
            r64 = [_bits_to_cuda(synth.make_router(w4n, args.seed, xs64[l], layer=l)) for l in range(8)]
            fx64 = [_bits_to_cuda(x) for x in xs64]
            K64 = 8 * 25
            ms64, _ = run_chain(st64, r64, w4n.T, K64, 16, fixed_inputs=fx64)
            ms64 = _max_over_ranks(ms64)
            k_ms, k_bytes, k_flops, ids64 = kernel_timing(st64, r64, w4n.T, 16, fixed_inputs=fx64)
            sb64 = np.mean([step_bytes(w4n, ids64[i], wd) for i in range(ids64.shape[0])])
            tf_peak, tf_kind = _tensor_peak(wd)
            extras["batch64"][wd] = {
                "workload": f"cfg4: 64 tokens, Zipf(1.1)-skewed routing, {wd} weights, tensor-core path",
                "tokens_per_s": world * w4n.T * K64 / (ms64 / 1e3), "us_per_layer": ms64 / K64 * 1e3,
                "step_bytes": sb64, "achieved_gbs": sb64 / (ms64 / K64 / 1e3) / 1e9,
                "frac_of_peak": sb64 / (ms64 / K64 / 1e3) / 1e9 / peak,
                "union_experts_mean": float(np.mean([len(np.unique(ids64[i])) for i in range(ids64.shape[0])])),
                "gateup_kernel": {"name": "k_mma_ffn<gate/up>", "us": k_ms * 1e3, "bytes": k_bytes,
                                  "gbs": k_bytes / (k_ms / 1e3) / 1e9,
                                  "frac_of_hbm_peak": k_bytes / (k_ms / 1e3) / 1e9 / peak,
                                  "tflops": k_flops / (k_ms / 1e3) / 1e12,
                                  "frac_of_tensor_peak": k_flops / (k_ms / 1e3) / 1e12 / tf_peak,
                                  "tensor_peak_tflops": tf_peak, "tensor_peak_kind": tf_kind}}
            del st64, fx64, r64
            torch.cuda.empty_cache()
        extras["lm_head"] = run_lm_head(world)
        extras["prefill"] = run_prefill(world, args.seed)
        extras["attn_prologue"] = run_attn_prologue(args.seed)
        extras["decode_attention"] = run_decode_attention(args.seed)
        extras["ep_emulated"] = run_ep(args.seed)
        extras["stack47"] = {
            "workload": "cfg3: 47 resident layers (21.4 GB NVFP4), residual chain, no attention",
            "batch1_tokens_per_s": tok_s / N_LAYERS, "batch1_us_per_layer": ms_step * 1e3,
            "batch4_tokens_per_s": world * w4.T * K4 / (ms4 / 1e3) / N_LAYERS,
            "batch4_us_per_layer": ms4 / K4 * 1e3, "batch4_step_bytes": b4_bytes,
            "batch4_frac_of_peak": b4_bytes / (ms4 / K4 / 1e3) / 1e9 / peak}

    if rank == 0:
        achieved = step_gbs
        line = {
            "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 x f16 -> f32",
            "data": "synthetic (seeded N(0,0.02) weights quantised to NVFP4, N(0,1) bf16 activations)",
            "config": {"workload": "cfg1: Flint-shaped MoE layer, d=2048, I=512, 256 routed + 1 shared experts, "
                                   "top-6, NVFP4 weights (W4A16), decode batch 1",
                       "global_batch": world, "seq_len": 1, "parallelism": f"replicas x{world}",
                       "step": "one layer call: route + top-6 + group + gate/up + down + combine",
                       "l2": "inputs larger than L2: 47 resident layer weight sets (21.4 GB) used in turn, "
                             "each step's output feeding the next (residual chain, input RMS-normalised "
                             "inside the layer so the chain stays finite)",
                       "launch": "CUDA graphs of layer calls chained with programmatic dependent launch, one "
                                 "launch of the batch-1 cluster kernel (7 clusters of 16 CTAs) per call",
                       "arithmetic": "e2m1*e4m3 weights exact in f16, x scaled by a power of two into f16, "
                                     "products exact, fp32 accumulation; bf16 output",
                       "weights": "nvfp4", "activations": "bf16", "accumulate": "f32"},
            "hbm": {"step_bytes": sb, "achieved_gbs": step_gbs, "frac_of_8tbs": step_gbs / NOMINAL_HBM_GBS,
                    "frac_of_peak": step_gbs / peak, "peak_gbs": peak, "peak_kind": peak_kind,
                    "router_bytes_excluded": w1.E * w1.d * 2},
            "roofline": {"bound": "hbm", "kernel": "k_tok1", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": TRAFFIC_K_TOK1, "peak_kind": peak_kind,
                         "kernel_us": ms_step * 1e3, "algorithmic_bytes": sb,
                         "timing": "CUDA events around the graph replays of the timed region; one launch "
                                   "per step"},
            "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": K,
            "clocks": clocks,
        }
        line.update(extras)
        if world == 1:
            line["cpu_baseline"] = cpu_baseline(seed=args.seed)
        print(json.dumps(line), flush=True)
    if _DIST["on"]:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_profile_case(args):
    """A small, self-contained case for ncu: one Flint-shaped layer (0.46 GB
    NVFP4 or 1.6 GB bf16 on the device) and `--steps` eager layer calls."""
    import torch
    import nvfp4_weight_only_flint_b200 as fm
    fm.lib()
    if args.profile == "attn":
        return run_profile_attn(args)
    if args.profile == "prefill":  # 8192 tokens, the Flint shape, NVFP4 (1.5 GB with the workspace)
        w = synth.CONFIGS["cfg1"]
        T = 8192
        st = Stack(w, 1, args.seed, max_tokens=T)
        xb = synth.x_bits(args.seed + 3000, T, w.d)
        x = _bits_to_cuda(xb)
        wr = _bits_to_cuda(synth.to_bf16_bits(synth.router_plain(args.seed, w.d, w.E, 0)))
    else:
        name = {"t1": "cfg1", "t8": "cfg2", "t64_nvfp4": "cfg4_nvfp4", "t64_bf16": "cfg4_bf16"}[args.profile]
        w = synth.CONFIGS[name]
        T = w.T
        st = Stack(synth.CONFIGS["cfg1"], 1, args.seed, max_tokens=T, wdtype=w.wdtype)
        xb = synth.x_bits(args.seed + 3000, T, w.d)
        x = _bits_to_cuda(xb)
        wr = _bits_to_cuda(synth.make_router(w, args.seed, xb))
    out = torch.empty_like(x)
    opt = fm.Options(path=fm.FLINT_PATH_AUTO, use_pdl=1)
    for _ in range(max(1, args.steps)):
        fm.flint_moe_forward_ex(x, T, wr, st.layers[0][3], st.shape, None, out, st.ws, opt)
    torch.cuda.synchronize()
    rc, flags = fm.flint_moe_get_status(st.ws)
    if rc != 0:
        raise RuntimeError(f"device status {rc} flags {flags}")
    return 0


def run_profile_attn(args):
    """Small case for ncu of the attention kernels: the prologue over 8192
    tokens, decode attention of 8 tokens over 32K cache rows each and of one
    token over 32K rows (about 0.9 GB on the device), `--steps` eager calls
    of each."""
    import torch
    import nvfp4_weight_only_flint_b200 as fm
    hq, hkv, dh, T, L, Tp = 32, 4, 128, 8, 32768, 8192
    g = torch.Generator(device="cuda").manual_seed(args.seed)
    kc = torch.randn((T * L, hkv, dh), device="cuda", generator=g).to(torch.bfloat16)
    vc = torch.randn((T * L, hkv, dh), device="cuda", generator=g).to(torch.bfloat16)
    q = torch.randn((T, hq, dh), device="cuda", generator=g).to(torch.bfloat16)
    out = torch.empty_like(q)
    start = torch.arange(T, device="cuda", dtype=torch.int64) * L
    length = torch.full((T,), L, device="cuda", dtype=torch.int32)
    nb = fm.flint_decode_attention_workspace_bytes(T, hkv, L)
    ws = torch.empty(max(nb, 16), device="cuda", dtype=torch.uint8)
    ws1 = torch.empty(max(fm.flint_decode_attention_workspace_bytes(1, hkv, L), 16), device="cuda",
                      dtype=torch.uint8)
    qkv = torch.randn((Tp, hq + 2 * hkv, dh), device="cuda", generator=g).to(torch.bfloat16)
    w1 = torch.ones(dh, device="cuda").to(torch.bfloat16)
    cs = torch.zeros((Tp, dh), device="cuda", dtype=torch.float32)
    cs[:, : dh // 2] = 1.0
    pos = torch.arange(Tp, device="cuda", dtype=torch.int32)
    q_out = torch.empty((Tp, hq, dh), device="cuda", dtype=torch.bfloat16)
    status = torch.zeros(1, device="cuda", dtype=torch.int32)
    for _ in range(max(1, args.steps)):
        fm.flint_qk_norm_rope_kv(qkv, Tp, hq, hkv, w1, w1, cs, Tp, pos, True, 1e-6, pos, T * L, q_out, kc, vc,
                                 status)
        fm.flint_decode_attention(q, kc, vc, T * L, start, length, T, hq, hkv, L, dh ** -0.5, out, ws, status)
        fm.flint_decode_attention(q, kc, vc, T * L, start, length, 1, hq, hkv, L, dh ** -0.5, out, ws1, status)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device check flags {int(status.item())}")
    return 0


def run_reference(args, world):
    """Reference arm: the fp64 oracle on the host cores, steps of one
    single-token layer decode each (bounded sample)."""
    import oracle
    w = synth.CONFIGS["cfg1"]
    cores = _host_cores()
    K = min(args.steps, 12)             # a bounded sample: ~0.1 s of fp64 work per step
    W = max(3, min(args.warmup, 5))     # at least 3 warm-up steps, as for the GPU arm
    prepared = []
    for i in range(K + W):
        x = synth.x_bits(args.seed + 50 + i, 1, w.d)
        wr = synth.make_router(w, args.seed, x, layer=i % N_LAYERS)
        ids, _, _ = oracle.topk(oracle.router_logits(x, wr), w.k)
        experts = [None] * (w.E + w.S)
        for e in list(ids[0]) + list(range(w.E, w.E + w.S)):
            g, u, dn = synth.expert_weights_np(args.seed, i % N_LAYERS, int(e), w.d, w.inter, w.std)
            experts[int(e)] = (oracle.quantize(g), oracle.quantize(u), oracle.quantize(dn))
        prepared.append((x, wr, experts))
    for x, wr, ex in prepared[:W]:
        oracle.moe_forward(x, wr, ex, d=w.d, inter=w.inter, E=w.E, k=w.k, S=w.S, n_threads=cores)
    t0 = time.perf_counter()
    for x, wr, ex in prepared[W:]:
        oracle.moe_forward(x, wr, ex, d=w.d, inter=w.inter, E=w.E, k=w.k, S=w.S, n_threads=cores)
    dt = time.perf_counter() - t0
    val = K / dt
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": dt / K * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "cfg1: Flint-shaped MoE layer, d=2048, I=512, 256 routed + 1 shared experts, "
                                   "top-6, NVFP4 weights (W4A16), decode batch 1"},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": min(cores, w.k + w.S), "kind": "oracle",
                             "host_threads": cores,
                             "sample": f"{K} single-token layer decodes (fp64 oracle, {cores} threads offered, one "
                                       f"busy per expert job: {min(cores, w.k + w.S)}), expert quantisation untimed"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


import ctypes  # noqa: E402

ctypes_void_p = ctypes.c_void_p
ctypes_addressof = ctypes.addressof

if __name__ == "__main__":
    sys.exit(main())
