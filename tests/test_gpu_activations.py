"""Activations with a wide dynamic range on every path. bf16 allows values
from about 1e-38 to 3e38 in one token; the NVFP4 paths stage x (and h) in f16
after a per-token (per-row) power-of-two scale, so a token holding both 1e3
and 1e-4 must still match the fp64 oracle within the layer tolerance: rows of
mixed magnitude, a token scaled by 1e-3, one by 3e3, one with values near the
f16 staging limit (6e4)."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import GpuLayer, bits_to_cuda, check_output, check_routing, cuda_to_bits

pytestmark = pytest.mark.gpu

_L = {}


def _layer(wdtype, T):
    key = (wdtype,)
    if key not in _L:
        _L[key] = GpuLayer(synth.CONFIGS["cfg1"], seed=23, max_tokens=64, keep_f32=False, wdtype=wdtype)
    return _L[key]


def wide_tokens(T, d, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d)).astype(np.float32)
    for t in range(T):
        kind = t % 4
        if kind == 0:    # a few large and a few tiny entries among N(0, 1)
            idx = rng.choice(d, 8, replace=False)
            x[t, idx[:4]] = np.array([1e3, -1e3, 5e2, -2e2], np.float32)
            x[t, idx[4:]] = np.array([1e-4, -3e-5, 2e-4, 7e-5], np.float32)
        elif kind == 1:  # a small token
            x[t] *= 1e-3
        elif kind == 2:  # a large token
            x[t] *= 3e3
        else:            # entries near the f16 staging limit
            idx = rng.choice(d, 3, replace=False)
            x[t, idx] = np.array([6e4, -5e4, 3e4], np.float32)
    return synth.to_bf16_bits(x)


@pytest.mark.parametrize("T,wdtype,variant,path", [
    (1, "nvfp4", fm.FLINT_LAYER_AUTO, fm.FLINT_PATH_AUTO),      # cluster kernel
    (1, "nvfp4", fm.FLINT_LAYER_FMA, fm.FLINT_PATH_AUTO),       # persistent kernel, CUDA cores
    (4, "nvfp4", fm.FLINT_LAYER_MMA, fm.FLINT_PATH_AUTO),       # persistent kernel, mma.sync
    (4, "nvfp4", fm.FLINT_LAYER_FMA, fm.FLINT_PATH_AUTO),
    (12, "nvfp4", fm.FLINT_LAYER_AUTO, fm.FLINT_PATH_AUTO),     # three-kernel path
    (40, "nvfp4", fm.FLINT_LAYER_AUTO, fm.FLINT_PATH_AUTO),     # tcgen05 path
    (40, "bf16", fm.FLINT_LAYER_AUTO, fm.FLINT_PATH_AUTO),      # tcgen05 path, bf16 weights
])
def test_wide_range_activations(T, wdtype, variant, path):
    w = synth.CONFIGS["cfg1"]
    layer = _layer(wdtype, T)
    for s in range(4 if T == 1 else 1):
        x_bits = wide_tokens(T, w.d, 500 + 10 * T + s)
        if T == 1:
            x_bits = wide_tokens(4, w.d, 500 + s)[s:s + 1].copy()  # each of the four kinds alone
        wr_bits = synth.make_router(w, 500 + T + s, x_bits)
        out, ids, gates = layer.forward(bits_to_cuda(x_bits), bits_to_cuda(wr_bits), path=path, variant=variant)
        torch.cuda.synchronize()
        ids_np = ids.cpu().numpy()
        check_routing(ids_np, gates.cpu().numpy(), oracle.router_logits(x_bits, wr_bits), w.k)
        ref = layer.oracle_forward(x_bits, wr_bits, ids_np)
        # per token, so a large token cannot hide a small one's error
        for t in range(T):
            check_output(cuda_to_bits(out)[t:t + 1], ref["out"][t:t + 1], f"T={T} {wdtype} token {t} kind {t % 4}")
        assert fm.flint_moe_get_status(layer.ws) == (0, 0)
