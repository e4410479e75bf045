"""Parity of the batch-2..8 cluster kernel (persistent 16-CTA clusters taking the
selected experts in turn, register-fragment tensor cores) against the fp64
oracle: the Flint shape at every batch from 2 to 8, the overlapping-routing
workload at batch 8, shape variants, residual and input norm, many consecutive
launches (arrival counters back at zero, bitwise-reproducible output), its
agreement with the persistent kernel, and the shapes it refuses."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import synth
from gpu_layer import GpuLayer, bits_to_cuda, check_output, check_routing, cuda_to_bits
import oracle

pytestmark = pytest.mark.gpu

CLUSTER = fm.FLINT_LAYER_CLUSTER
_LAYER = {}


def _flint_layer(name="cfg2"):
    if name not in _LAYER:
        _LAYER[name] = GpuLayer(synth.CONFIGS[name], seed=13, max_tokens=8, keep_f32=False)
    return _LAYER[name]


def _check(layer, x_bits, wr_bits, residual_bits=None, input_norm=False, what="", variant=CLUSTER):
    x, wr = bits_to_cuda(x_bits), bits_to_cuda(wr_bits)
    res = bits_to_cuda(residual_bits) if residual_bits is not None else None
    out, ids, gates = layer.forward(x, wr, residual=res, input_norm=input_norm, variant=variant)
    torch.cuda.synchronize()
    ids_np, gates_np = ids.cpu().numpy(), gates.cpu().numpy()
    logits = oracle.router_logits(x_bits, wr_bits)
    if input_norm:
        xf = synth.bf16_bits_to_f64(x_bits)
        logits = logits / np.sqrt(np.mean(xf ** 2, axis=1, keepdims=True) + 1e-6)
    check_routing(ids_np, gates_np, logits, layer.w.k)
    ref = layer.oracle_forward(x_bits, wr_bits, ids_np, residual_bits=residual_bits, input_norm=input_norm)
    check_output(cuda_to_bits(out), ref["out"], what)
    assert fm.flint_moe_get_status(layer.ws) == (0, 0)
    return out, ids_np


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tokn_overlapping_routing_batch8(seed):
    # tokens share about 40 % of their experts: items carry 1..8 tokens
    w = synth.CONFIGS["cfg2"]
    layer = _flint_layer()
    x = synth.x_bits(300 + seed, 8, w.d)
    _check(layer, x, synth.make_router(w, 300 + seed, x), what=f"cfg2 seed {seed}")


@pytest.mark.parametrize("T", [2, 3, 4, 5, 6, 7, 8])
def test_tokn_every_batch(T):
    w = synth.CONFIGS["cfg2"]
    layer = _flint_layer()
    x = synth.x_bits(310 + T, T, w.d)
    _check(layer, x, synth.make_router(w, 310 + T, x), what=f"T={T}")


def test_tokn_all_tokens_one_expert_set():
    # every token picks the same experts: 7 items of 8 tokens each
    w = synth.CONFIGS["cfg2"]
    layer = _flint_layer()
    x1 = synth.x_bits(320, 1, w.d)
    x = np.repeat(x1, 8, axis=0)
    _check(layer, x, synth.make_router(w, 320, x1), what="identical tokens")


def test_tokn_residual_and_input_norm():
    w = synth.CONFIGS["cfg2"]
    layer = _flint_layer()
    x = synth.x_bits(330, 6, w.d)
    res = synth.x_bits(331, 6, w.d)
    wr = synth.make_router(w, 330, x)
    _check(layer, x, wr, residual_bits=res, what="residual")
    _check(layer, x, wr, residual_bits=res, input_norm=True, what="residual + input norm")
    # one token scaled far up, one far down: per-token staging scales
    xf = synth.bf16_bits_to_f64(x).astype(np.float32)
    xf[0] *= 300.0
    xf[1] *= 1e-3
    _check(layer, synth.to_bf16_bits(xf), wr, input_norm=True, what="mixed magnitudes")


def test_tokn_agrees_with_persistent_kernel():
    w = synth.CONFIGS["cfg2"]
    layer = _flint_layer()
    x = synth.x_bits(340, 8, w.d)
    wr = synth.make_router(w, 340, x)
    a, ids_a = _check(layer, x, wr, what="cluster")
    b, ids_b = _check(layer, x, wr, what="persistent, tensor cores", variant=fm.FLINT_LAYER_MMA)
    assert np.array_equal(ids_a, ids_b)
    da, db = synth.bf16_bits_to_f64(cuda_to_bits(a)), synth.bf16_bits_to_f64(cuda_to_bits(b))
    assert np.linalg.norm(da - db) <= 5e-3 * np.linalg.norm(db)


def test_tokn_many_launches_deterministic():
    w = synth.CONFIGS["cfg2"]
    layer = _flint_layer()
    x_bits = synth.x_bits(350, 8, w.d)
    wr_bits = synth.make_router(w, 350, x_bits)
    x, wr = bits_to_cuda(x_bits), bits_to_cuda(wr_bits)
    first, _, _ = layer.forward(x, wr, variant=CLUSTER)
    out = torch.empty_like(x)
    opt = fm.Options(path=fm.FLINT_PATH_AUTO, use_pdl=1, layer_variant=CLUSTER)
    for _ in range(499):
        fm.flint_moe_forward_ex(x, 8, wr, layer.weights, layer.shape, None, out, layer.ws, opt)
    nopdl, _, _ = layer.forward(x, wr, variant=CLUSTER, pdl=False)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), out.view(torch.int16))
    assert torch.equal(first.view(torch.int16), nopdl.view(torch.int16))
    assert fm.flint_moe_get_status(layer.ws) == (0, 0)
    assert not layer.ws[64:128].cpu().numpy().any()
    _check(layer, x_bits, wr_bits, what="after 500 launches")


def test_tokn_then_tok1_share_counters():
    # batch 1 and batch 8 alternate on one workspace: both leave the shared
    # per-row-block counters at zero
    w = synth.CONFIGS["cfg2"]
    layer = _flint_layer()
    for i in range(3):
        x8 = synth.x_bits(360 + i, 8, w.d)
        _check(layer, x8, synth.make_router(w, 360 + i, x8), what=f"batch 8 #{i}")
        x1 = synth.x_bits(370 + i, 1, w.d)
        _check(layer, x1, synth.make_router(synth.CONFIGS["cfg1"], 370 + i, x1), what=f"batch 1 #{i}")
    assert not layer.ws[64:128].cpu().numpy().any()


@pytest.mark.parametrize("d,inter,E,k,S,T", [(512, 256, 32, 6, 1, 4), (512, 1024, 8, 8, 0, 8),
                                             (1024, 256, 64, 4, 1, 3), (1024, 512, 16, 2, 1, 8),
                                             (1024, 1024, 16, 3, 1, 5), (2048, 256, 40, 6, 0, 7),
                                             (2048, 512, 13, 6, 1, 2), (2048, 512, 256, 1, 0, 8)])
def test_tokn_shape_variants(d, inter, E, k, S, T):
    w = synth.Workload("var", d=d, inter=inter, E=E, k=k, S=S, T=T)
    layer = GpuLayer(w, seed=d + inter + E + T, max_tokens=8)
    for s in range(2):
        x = synth.x_bits(E + 17 * s, T, d)
        wr = synth.to_bf16_bits(np.random.default_rng(E + s).standard_normal((E, d)) * 0.02)
        _check(layer, x, wr, what=f"shape {d},{inter},{E},{k},{S} T={T} seed {s}")


def test_tokn_refuses_and_auto_falls_back():
    # inter=128 is below the kernel's 256-column down stages; E=512 above its
    # 256 router rows: the forced variant is refused, AUTO takes the
    # persistent kernel
    for (d, inter, E) in [(1024, 128, 16), (1024, 256, 512)]:
        w = synth.Workload("small", d=d, inter=inter, E=E, k=4, S=1, T=4)
        layer = GpuLayer(w, seed=5, max_tokens=8)
        x = synth.x_bits(5, 4, d)
        wr = synth.to_bf16_bits(np.random.default_rng(5).standard_normal((E, d)) * 0.02)
        with pytest.raises(fm.FlintError) as ei:
            layer.forward(bits_to_cuda(x), bits_to_cuda(wr), variant=CLUSTER)
        assert ei.value.code == -2
        _check(layer, x, wr, what=f"auto fallback d={d} inter={inter} E={E}", variant=fm.FLINT_LAYER_AUTO)
