"""Parity of the batch-1 cluster kernel (one 16-CTA cluster per selected expert
and one for the shared expert) against the fp64 oracle, at the Flint shape and
at shape variants (one expert, eight of eight experts, no shared expert, E not
a multiple of the cluster size, E = 512), with residual and input norm, over
many consecutive launches (its per-row-block arrival counters return to zero),
and its agreement with the persistent kernel's CUDA-core variant."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import GpuLayer, bits_to_cuda, check_output, check_routing, cuda_to_bits

pytestmark = pytest.mark.gpu

CLUSTER = fm.FLINT_LAYER_CLUSTER
_LAYER = {}


def _flint_layer():
    if "cfg1" not in _LAYER:
        _LAYER["cfg1"] = GpuLayer(synth.CONFIGS["cfg1"], seed=11, max_tokens=8, keep_f32=False)
    return _LAYER["cfg1"]


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


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_cluster_kernel_flint_shape(seed):
    w = synth.CONFIGS["cfg1"]
    layer = _flint_layer()
    x = synth.x_bits(200 + seed, 1, w.d)
    _check(layer, x, synth.make_router(w, 200 + seed, x), what=f"cluster kernel seed {seed}")


def test_cluster_kernel_residual_and_input_norm():
    w = synth.CONFIGS["cfg1"]
    layer = _flint_layer()
    x = synth.x_bits(210, 1, w.d)
    res = synth.x_bits(211, 1, w.d)
    wr = synth.make_router(w, 210, x)
    _check(layer, x, wr, residual_bits=res, what="residual")
    _check(layer, x, wr, residual_bits=res, input_norm=True, what="residual + input norm")
    # a large-magnitude token: the input norm and the f16 staging scale both act
    big = (synth.bf16_bits_to_f64(x) * 300.0).astype(np.float32)
    _check(layer, synth.to_bf16_bits(big), wr, input_norm=True, what="x * 300, input norm")


def test_cluster_kernel_agrees_with_persistent_kernel():
    w = synth.CONFIGS["cfg1"]
    layer = _flint_layer()
    x = synth.x_bits(220, 1, w.d)
    wr = synth.make_router(w, 220, x)
    a, ids_a = _check(layer, x, wr, what="cluster")
    b, ids_b = _check(layer, x, wr, what="persistent, CUDA-core", variant=fm.FLINT_LAYER_FMA)
    assert np.array_equal(ids_a, ids_b)
    da, db = synth.bf16_bits_to_f64(cuda_to_bits(a)), synth.bf16_bits_to_f64(cuda_to_bits(b))
    assert np.linalg.norm(da - db) <= 5e-3 * np.linalg.norm(db)


def test_cluster_kernel_many_launches_deterministic():
    # the per-row-block arrival counters must return to zero after every
    # launch; the fixed slot order of the final sum makes the output bitwise
    # reproducible, with or without programmatic dependent launch
    w = synth.CONFIGS["cfg1"]
    layer = _flint_layer()
    x_bits = synth.x_bits(230, 1, w.d)
    x, wr = bits_to_cuda(x_bits), bits_to_cuda(synth.make_router(w, 230, x_bits))
    first, _, _ = layer.forward(x, wr, variant=CLUSTER)
    out = torch.empty_like(x)
    opt = fm.Options(path=fm.FLINT_PATH_AUTO, use_pdl=1, layer_variant=CLUSTER)
    for _ in range(999):
        fm.flint_moe_forward_ex(x, 1, wr, layer.weights, layer.shape, None, out, layer.ws, opt)
    nopdl, _, _ = layer.forward(x, wr, variant=CLUSTER, pdl=False)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), out.view(torch.int16))
    assert torch.equal(first.view(torch.int16), nopdl.view(torch.int16))
    assert fm.flint_moe_get_status(layer.ws) == (0, 0)
    counters = layer.ws[64:128].cpu().numpy()
    assert not counters.any()
    _check(layer, x_bits, synth.make_router(w, 230, x_bits), what="after 1000 launches")


@pytest.mark.parametrize("d,inter,E,k,S", [(512, 128, 1, 1, 0), (512, 128, 8, 8, 1), (1024, 256, 64, 4, 1),
                                           (2048, 128, 40, 6, 0), (1024, 1024, 16, 3, 1),
                                           (2048, 512, 13, 6, 1), (2048, 512, 512, 8, 1),
                                           (512, 256, 256, 6, 1)])
def test_cluster_kernel_shape_variants(d, inter, E, k, S):
    w = synth.Workload("var", d=d, inter=inter, E=E, k=k, S=S, T=1)
    layer = GpuLayer(w, seed=d + inter + E + 7, max_tokens=1)
    for s in range(2):
        x = synth.x_bits(E + s, 1, d)
        wr = synth.to_bf16_bits(np.random.default_rng(E + s).standard_normal((E, d)) * 0.02)
        _check(layer, x, wr, what=f"shape {d},{inter},{E},{k},{S} seed {s}")


def test_cluster_kernel_after_other_expert_counts():
    # one kernel instantiation serves every E up to 256 (and another up to
    # 512): calls at E = 13, then 256, then 13 again at the same (d, inter)
    # must all launch (the shared-memory limit is the function's, not the
    # first call's)
    for E in (13, 256, 13, 40):
        w = synth.Workload("var", d=2048, inter=512, E=E, k=6, S=1, T=1)
        layer = GpuLayer(w, seed=E + 1, max_tokens=1, keep_f32=False)
        x = synth.x_bits(E + 3, 1, 2048)
        wr = synth.to_bf16_bits(np.random.default_rng(E + 3).standard_normal((E, 2048)) * 0.02)
        _check(layer, x, wr, what=f"E={E}")
        del layer
        torch.cuda.empty_cache()


def test_cluster_kernel_refuses_shapes_it_cannot_hold():
    # d=4096, inter=1024: a CTA's slice of one expert is 432 KB, above the
    # shared memory of an SM; the forced variant is refused, AUTO falls back
    w = synth.Workload("big", d=4096, inter=1024, E=12, k=2, S=1, T=1)
    layer = GpuLayer(w, seed=3, max_tokens=1)
    x = synth.x_bits(3, 1, 4096)
    wr = synth.to_bf16_bits(np.random.default_rng(3).standard_normal((12, 4096)) * 0.02)
    with pytest.raises(fm.FlintError) as ei:
        layer.forward(bits_to_cuda(x), bits_to_cuda(wr), variant=CLUSTER)
    assert ei.value.code == -2
    _check(layer, x, wr, what="auto fallback", variant=fm.FLINT_LAYER_AUTO)


def test_cluster_kernels_reject_more_than_eight_tokens():
    layer = _flint_layer()
    x = bits_to_cuda(synth.x_bits(240, 9, 2048))
    wr = bits_to_cuda(synth.make_router(synth.CONFIGS["cfg1"], 240, synth.x_bits(240, 1, 2048)))
    with pytest.raises(fm.FlintError) as ei:
        layer.forward(x, wr, variant=CLUSTER)
    assert ei.value.code == -2
