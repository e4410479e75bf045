"""GPU layer forward parity against the fp64 oracle: relative L2 <= 5e-3 and
max-abs <= 2e-2 * rms(out) for bf16 outputs; routed ids bit-exact (near ties
reported); edge cases (ragged token counts, zero input, single expert, shape
variants, residual), determinism, and the device wait-timeout check."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import GpuLayer, bits_to_cuda, check_output, check_routing, cuda_to_bits

pytestmark = pytest.mark.gpu

_LAYERS = {}


def _layer(name, seed=0, **kw):
    key = (name, seed, tuple(sorted(kw.items())))
    if key not in _LAYERS:
        _LAYERS.clear()
        torch.cuda.empty_cache()
        _LAYERS[key] = GpuLayer(synth.CONFIGS[name] if isinstance(name, str) else name, seed=seed, **kw)
    return _LAYERS[key]


def _run_and_check(layer, x_bits, wr_bits, residual_bits=None, path=fm.FLINT_PATH_AUTO, what="", split=False,
                   variant=fm.FLINT_LAYER_AUTO):
    x, wr = bits_to_cuda(x_bits), bits_to_cuda(wr_bits)
    res = bits_to_cuda(residual_bits) if residual_bits is not None else None
    out, ids, gates = layer.forward(x, wr, residual=res, path=path, split=split, variant=variant)
    torch.cuda.synchronize()
    ids_np, gates_np = ids.cpu().numpy(), gates.cpu().numpy()
    near = check_routing(ids_np, gates_np, oracle.router_logits(x_bits, wr_bits), layer.w.k)
    ref = layer.oracle_forward(x_bits, wr_bits, ids_np, residual_bits=residual_bits)
    rel, mx = check_output(cuda_to_bits(out), ref["out"], what)
    assert fm.flint_moe_get_status(layer.ws) == (0, 0)
    return out, ids_np, near, rel


def test_forward_cfg0():
    w = synth.CONFIGS["cfg0"]
    layer = _layer("cfg0")
    for s in range(3):
        x = synth.x_bits(s, w.T, w.d)
        _run_and_check(layer, x, synth.make_router(w, s, x), what=f"cfg0 seed {s}")


def test_forward_cfg1_batch1():
    w = synth.CONFIGS["cfg1"]
    layer = _layer("cfg1", max_tokens=32)
    for s in range(3):
        x = synth.x_bits(s, 1, w.d)
        _run_and_check(layer, x, synth.make_router(w, s, x), what=f"cfg1 seed {s}")


def test_forward_cfg2_batch8_overlap():
    w = synth.CONFIGS["cfg2"]
    layer = _layer("cfg1", max_tokens=32)
    x = synth.x_bits(0, w.T, w.d)
    wr = synth.make_router(w, 0, x)
    _, ids, _, _ = _run_and_check(layer, x, wr, what="cfg2")
    assert 0.3 <= synth.overlap_fraction(ids) <= 0.5
    assert len(set(ids.ravel().tolist())) < w.T * w.k


@pytest.mark.parametrize("name,T", [("cfg1", 1), ("cfg2", 8), ("cfg0", 4)])
def test_forward_split_kernel_path(name, T):
    # batch <= 8 runs as one persistent kernel by default; the three-kernel
    # path must give the same results within the tolerance
    w = synth.CONFIGS[name]
    layer = _layer("cfg0" if name == "cfg0" else "cfg1", max_tokens=32)
    x = synth.x_bits(40 + T, T, w.d)
    wr = synth.make_router(w, 40, x)
    a, ids_a, _, _ = _run_and_check(layer, x, wr, what=f"{name} fused")
    b, ids_b, _, _ = _run_and_check(layer, x, wr, what=f"{name} split", split=True)
    assert np.array_equal(ids_a, ids_b)


@pytest.mark.parametrize("variant", [fm.FLINT_LAYER_FMA, fm.FLINT_LAYER_MMA])
@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_forward_single_kernel_variants(T, variant):
    # the persistent kernel's two inner-loop variants (CUDA-core dot products,
    # register-fragment tensor-core MMA) at batch 1..8, including batches
    # whose experts serve one token (7 of the 8 MMA columns unused)
    w = synth.CONFIGS["cfg1"]
    layer = _layer("cfg1", max_tokens=32)
    x = synth.x_bits(60 + T, T, w.d)
    _run_and_check(layer, x, synth.make_router(w, 60 + T, x), what=f"T={T} variant {variant}", variant=variant)


def test_forward_single_kernel_variants_agree():
    w = synth.CONFIGS["cfg2"]
    layer = _layer("cfg1", max_tokens=32)
    x = synth.x_bits(70, w.T, w.d)
    wr = synth.make_router(w, 70, x)
    a, ids_a, _, _ = _run_and_check(layer, x, wr, what="fma", variant=fm.FLINT_LAYER_FMA)
    b, ids_b, _, _ = _run_and_check(layer, x, wr, what="mma", variant=fm.FLINT_LAYER_MMA)
    assert np.array_equal(ids_a, ids_b)
    da, db = synth.bf16_bits_to_f64(cuda_to_bits(a)), synth.bf16_bits_to_f64(cuda_to_bits(b))
    assert np.linalg.norm(da - db) <= 5e-3 * np.linalg.norm(db)


def test_forward_mixed_batches_one_workspace():
    # batch sizes change from call to call on one workspace: the persistent
    # kernel's tagged logits and h sit at offsets that do not move with T
    w = synth.CONFIGS["cfg1"]
    layer = _layer("cfg1", max_tokens=32)
    for i, T in enumerate([1, 8, 3, 8, 1, 6, 2, 8]):
        x = synth.x_bits(90 + i, T, w.d)
        _run_and_check(layer, x, synth.make_router(w, 90 + i, x), what=f"call {i}, T={T}")


def test_forward_batch8_after_many_batch1():
    # the SwiGLU values travel between CTAs under a launch tag: a batch-8 call
    # after 4095 batch-1 calls (whose launches leave rows 7.. of the tagged h
    # untouched) must see only its own values
    w1, w8 = synth.CONFIGS["cfg1"], synth.CONFIGS["cfg2"]
    layer = _layer("cfg1", max_tokens=32)
    x = synth.x_bits(95, 8, w8.d)
    _run_and_check(layer, x, synth.make_router(w8, 95, x), what="batch 8, first")
    x1 = bits_to_cuda(synth.x_bits(96, 1, w1.d))
    wr1 = bits_to_cuda(synth.make_router(w1, 96, synth.x_bits(96, 1, w1.d)))
    out1 = torch.empty_like(x1)
    opt = fm.Options(path=fm.FLINT_PATH_AUTO, use_pdl=1)
    for _ in range(4095):
        fm.flint_moe_forward_ex(x1, 1, wr1, layer.weights, layer.shape, None, out1, layer.ws, opt)
    torch.cuda.synchronize()
    assert fm.flint_moe_get_status(layer.ws) == (0, 0)
    x = synth.x_bits(97, 8, w8.d)
    _run_and_check(layer, x, synth.make_router(w8, 97, x), what="batch 8, 4096 launches later")


@pytest.mark.parametrize("T", [2, 3, 5, 9, 13, 31])
def test_forward_ragged_tokens(T):
    w = synth.CONFIGS["cfg1"]
    layer = _layer("cfg1", max_tokens=32)
    x = synth.x_bits(100 + T, T, w.d)
    _run_and_check(layer, x, synth.make_router(w, T, x), what=f"T={T}")


def test_forward_residual_and_in_place_output():
    w = synth.CONFIGS["cfg1"]
    layer = _layer("cfg1", max_tokens=32)
    x_bits = synth.x_bits(7, 4, w.d)
    wr_bits = synth.make_router(w, 7, x_bits)
    res_bits = synth.x_bits(8, 4, w.d)
    out, ids, _, _ = _run_and_check(layer, x_bits, wr_bits, residual_bits=res_bits, what="residual")
    # out aliasing the residual buffer gives the same bytes
    res = bits_to_cuda(res_bits)
    out2, _, _ = layer.forward(bits_to_cuda(x_bits), bits_to_cuda(wr_bits), residual=res, out=res)
    torch.cuda.synchronize()
    assert np.array_equal(cuda_to_bits(out2), cuda_to_bits(out))


def test_forward_zero_input_gives_zero():
    w = synth.CONFIGS["cfg1"]
    layer = _layer("cfg1", max_tokens=32)
    x = np.zeros((3, w.d), np.uint16)
    wr = synth.make_router(w, 0, synth.x_bits(0, 1, w.d))
    out, ids, gates = layer.forward(bits_to_cuda(x), bits_to_cuda(wr))
    torch.cuda.synchronize()
    assert not cuda_to_bits(out).any() or np.all(synth.bf16_bits_to_f64(cuda_to_bits(out)) == 0)
    assert ids.cpu().numpy().tolist() == [[0, 1, 2, 3, 4, 5]] * 3


def test_forward_deterministic_and_pdl_invariant():
    w = synth.CONFIGS["cfg2"]
    layer = _layer("cfg1", max_tokens=32)
    x_bits = synth.x_bits(3, 8, w.d)
    wr = bits_to_cuda(synth.make_router(w, 3, x_bits))
    x = bits_to_cuda(x_bits)
    a, _, _ = layer.forward(x, wr, pdl=True)
    b, _, _ = layer.forward(x, wr, pdl=True)
    c, _, _ = layer.forward(x, wr, pdl=False)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


@pytest.mark.parametrize("variant", [fm.FLINT_LAYER_FMA, fm.FLINT_LAYER_MMA])
@pytest.mark.parametrize("d,inter,E,k,S,T", [(512, 128, 1, 1, 0, 3), (512, 128, 8, 8, 1, 5),
                                             (1024, 256, 64, 4, 1, 6), (4096, 1024, 12, 2, 1, 3),
                                             (2048, 128, 40, 6, 0, 4), (1024, 1024, 16, 3, 1, 2)])
def test_forward_shape_variants(d, inter, E, k, S, T, variant):
    w = synth.Workload("var", d=d, inter=inter, E=E, k=k, S=S, T=T)
    layer = GpuLayer(w, seed=d + inter + E, max_tokens=T)
    x = synth.x_bits(E, T, d)
    wr = synth.to_bf16_bits(np.random.default_rng(E).standard_normal((E, d)) * 0.02)
    _run_and_check(layer, x, wr, what=f"shape {d},{inter},{E},{k},{S} variant {variant}", variant=variant)


@pytest.mark.parametrize("T", [1, 4])
def test_forward_stack_cfg3_sampled_layers(T):
    # 47 layers with a residual between them (x_{l+1} = out_l, residual = x_l),
    # each layer's input RMS-normalised inside the layer (without it the chain
    # overflows: SwiGLU grows quadratically in x). Every layer's routing is
    # checked on the GPU's own input; the full output on sampled layers.
    w = synth.CONFIGS["cfg3_t4" if T == 4 else "cfg3_t1"]
    _LAYERS.clear()
    torch.cuda.empty_cache()
    layers = [GpuLayer(w, seed=0, layer=l, max_tokens=4, keep_f32=False) for l in range(w.layers)]
    routers = []
    x_bits = synth.x_bits(0, w.T, w.d)
    x = bits_to_cuda(x_bits)
    xs = [x_bits]
    outs = []
    ids_all = []
    for l, L in enumerate(layers):
        wr_bits = synth.make_router(w, 0, xs[0], layer=l)
        routers.append(wr_bits)
        out, ids, gates = L.forward(x, bits_to_cuda(wr_bits), residual=x, input_norm=True)
        torch.cuda.synchronize()
        ids_all.append((ids.cpu().numpy(), gates.cpu().numpy()))
        x = out
        outs.append(cuda_to_bits(out))
        xs.append(outs[-1])
    for l in range(w.layers):
        xf = synth.bf16_bits_to_f64(xs[l])
        xn_logits = oracle.router_logits(xs[l], routers[l]) / np.sqrt(np.mean(xf ** 2, axis=1, keepdims=True) + 1e-6)
        check_routing(ids_all[l][0], ids_all[l][1], xn_logits, w.k)
    for l in (0, 23, 46):
        ref = layers[l].oracle_forward(xs[l], routers[l], ids_all[l][0], residual_bits=xs[l], input_norm=True)
        check_output(outs[l], ref["out"], f"stack layer {l}")
        assert np.all(np.isfinite(synth.bf16_bits_to_f64(outs[l])))
    del layers
    torch.cuda.empty_cache()


def test_device_wait_timeout_is_reported_and_context_survives():
    w = synth.CONFIGS["cfg0"]
    layer = _layer("cfg0")
    fm.flint_debug_wait_timeout(layer.ws, 200000)
    rc, flags = fm.flint_moe_get_status(layer.ws)
    assert rc == -7 and flags & 4
    x = synth.x_bits(1, w.T, w.d)
    _run_and_check(layer, x, synth.make_router(w, 1, x), what="after timeout")
