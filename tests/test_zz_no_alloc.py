"""flint_moe_forward_noalloc: the layer forward for callers that cannot allocate
device memory at call time (its scratch is a fixed array compiled into the
library). Its output must match flint_moe_forward's, which uses a caller
workspace, within the parity tolerance, on two calls in a row (the second call
runs on scratch that still holds the first call's contents).

This file is collected last so that a stop-at-first-failure run has already run
every other test."""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import synth
from gpu_layer import MAX_ABS_TOL_RMS, REL_L2_TOL, GpuLayer, bits_to_cuda, cuda_to_bits

pytestmark = pytest.mark.gpu


def _close(a_bits, b_bits):
    a = synth.bf16_bits_to_f64(a_bits)
    b = synth.bf16_bits_to_f64(b_bits)
    rms = np.sqrt(np.mean(b ** 2))
    assert np.linalg.norm(a - b) <= REL_L2_TOL * np.linalg.norm(b)
    assert np.abs(a - b).max() <= MAX_ABS_TOL_RMS * rms


@pytest.mark.parametrize("name,T", [("cfg1", 1), ("cfg2", 8), ("cfg0", 4)])
def test_noalloc_matches_workspace_forward_twice(name, T):
    w = synth.CONFIGS[name]
    layer = GpuLayer(synth.CONFIGS["cfg0" if name == "cfg0" else "cfg1"], seed=5, max_tokens=T, keep_f32=False)
    x_bits = synth.x_bits(21, T, w.d)
    x = bits_to_cuda(x_bits)
    wr = bits_to_cuda(synth.make_router(w, 21, x_bits))
    res = bits_to_cuda(synth.x_bits(22, T, w.d))
    ref = torch.empty_like(x)
    fm.flint_moe_forward(x, T, wr, layer.weights, layer.shape, res, ref, layer.ws)
    outs = []
    for _ in range(2):
        out = torch.full_like(x, float("nan"))
        fm.flint_moe_forward_noalloc(x, T, wr, layer.weights, layer.shape, res, out)
        outs.append(out)
    torch.cuda.synchronize()
    ref_bits = cuda_to_bits(ref)
    for out in outs:
        _close(cuda_to_bits(out), ref_bits)


def test_noalloc_rejects_calls_beyond_its_scratch():
    # d=2048, I=1024, top-8 + shared at 31 tokens needs > 1 MiB of scratch;
    # the call is refused on the host before anything is launched.
    shape = fm.Shape(2048, 1024, 64, 8, 1, fm.FLINT_W_NVFP4)
    assert fm.flint_moe_workspace_bytes(shape, 31) > (1 << 20)
    w = fm.Weights(0x100000, 0x200000, 0x300000)
    rc = fm.lib().flint_moe_forward_noalloc(0x400000, 31, 0x500000, ctypes.byref(w), ctypes.byref(shape), None,
                                            0x600000, None)
    assert rc == -4
    assert "scratch" in fm.flint_last_error()
