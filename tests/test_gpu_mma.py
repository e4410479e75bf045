"""Tensor-core (batch >= 32) layer path against the fp64 oracle.

Config 4's Flint-shaped layer (d=2048, I=512, 256 routed + 1 shared, top-6) at
64 tokens with a Zipf(1.1) expert-popularity bias, with NVFP4 and with bf16
weights; ragged token counts (expert token counts that are not multiples of the
MMA's N granularity of 16, and the shared expert used by every token), the
path forced at small batch, the residual, and agreement with the GEMV path at
a batch both paths run. Same bar as the GEMV path: routed ids bit-exact (near
ties reported), relative L2 <= 5e-3 and max-abs <= 2e-2 * rms(out)."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import GpuLayer, bits_to_cuda, check_output, check_routing, cuda_to_bits

pytestmark = pytest.mark.gpu

_LAYERS = {}


def _layer(name, **kw):
    key = (name, tuple(sorted(kw.items())))
    if key not in _LAYERS:
        _LAYERS.clear()
        torch.cuda.empty_cache()
        _LAYERS[key] = GpuLayer(synth.CONFIGS[name], seed=0, **kw)
    return _LAYERS[key]


def _run_and_check(layer, x_bits, wr_bits, residual_bits=None, path=fm.FLINT_PATH_AUTO, what=""):
    x, wr = bits_to_cuda(x_bits), bits_to_cuda(wr_bits)
    res = bits_to_cuda(residual_bits) if residual_bits is not None else None
    out, ids, gates = layer.forward(x, wr, residual=res, path=path)
    torch.cuda.synchronize()
    ids_np, gates_np = ids.cpu().numpy(), gates.cpu().numpy()
    check_routing(ids_np, gates_np, oracle.router_logits(x_bits, wr_bits), layer.w.k)
    ref = layer.oracle_forward(x_bits, wr_bits, ids_np, residual_bits=residual_bits)
    rel, mx = check_output(cuda_to_bits(out), ref["out"], what)
    assert fm.flint_moe_get_status(layer.ws) == (0, 0)
    return out, ids_np, rel


@pytest.mark.parametrize("name", ["cfg4_nvfp4", "cfg4_bf16"])
def test_mma_cfg4_zipf_batch64(name):
    w = synth.CONFIGS[name]
    layer = _layer(name, max_tokens=128, keep_f32=False)
    x = synth.x_bits(0, w.T, w.d)
    wr = synth.make_router(w, 0, x)
    _, ids, _ = _run_and_check(layer, x, wr, what=name)
    counts = np.bincount(ids.ravel(), minlength=w.E)
    # the Zipf bias skews the selections: some expert serves many tokens, and
    # many serve one, so the grouped tiles are ragged
    assert counts.max() >= 16 and (counts == 1).sum() >= 10


@pytest.mark.parametrize("T", [32, 33, 47, 100, 128])
def test_mma_ragged_token_counts(T):
    w = synth.CONFIGS["cfg4_nvfp4"]
    layer = _layer("cfg4_nvfp4", max_tokens=128, keep_f32=False)
    x = synth.x_bits(100 + T, T, w.d)
    _run_and_check(layer, x, synth.make_router(w, 100 + T, x), what=f"T={T}")


@pytest.mark.parametrize("T", [1, 5, 16])
def test_mma_forced_at_small_batch(T):
    w = synth.CONFIGS["cfg1"]
    layer = _layer("cfg4_nvfp4", max_tokens=128, keep_f32=False)
    x = synth.x_bits(200 + T, T, w.d)
    _run_and_check(layer, x, synth.make_router(w, 200 + T, x), path=fm.FLINT_PATH_MMA, what=f"forced T={T}")


def test_mma_and_gemv_paths_agree():
    w = synth.CONFIGS["cfg1"]
    layer = _layer("cfg4_nvfp4", max_tokens=128, keep_f32=False)
    T = 24
    x = synth.x_bits(300, T, w.d)
    wr = synth.make_router(w, 300, x)
    a, ids_a, _ = _run_and_check(layer, x, wr, path=fm.FLINT_PATH_MMA, what="mma")
    b, ids_b, _ = _run_and_check(layer, x, wr, path=fm.FLINT_PATH_GEMV, what="gemv")
    assert np.array_equal(ids_a, ids_b)
    da, db = synth.bf16_bits_to_f64(cuda_to_bits(a)), synth.bf16_bits_to_f64(cuda_to_bits(b))
    assert np.linalg.norm(da - db) <= 5e-3 * np.linalg.norm(db)


@pytest.mark.parametrize("name", ["cfg4_nvfp4", "cfg4_bf16"])
def test_mma_residual_and_determinism(name):
    w = synth.CONFIGS[name]
    layer = _layer(name, max_tokens=128, keep_f32=False)
    x = synth.x_bits(400, w.T, w.d)
    res = synth.x_bits(401, w.T, w.d)
    wr = synth.make_router(w, 400, x)
    a, _, _ = _run_and_check(layer, x, wr, residual_bits=res, what=f"{name} residual")
    b, _, _ = _run_and_check(layer, x, wr, residual_bits=res, what=f"{name} residual again")
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_mma_zero_input_gives_residual():
    w = synth.CONFIGS["cfg4_nvfp4"]
    layer = _layer("cfg4_nvfp4", max_tokens=128, keep_f32=False)
    x = np.zeros((w.T, w.d), np.uint16)
    res = synth.x_bits(500, w.T, w.d)
    wr = synth.to_bf16_bits(synth.router_plain(500, w.d, w.E, 0))
    out, ids, _ = layer.forward(bits_to_cuda(x), bits_to_cuda(wr), residual=bits_to_cuda(res))
    torch.cuda.synchronize()
    # all logits are 0: the lowest ids win the ties, and every expert output is 0
    assert (ids.cpu().numpy() == np.arange(w.k)).all()
    assert np.array_equal(cuda_to_bits(out), res)
