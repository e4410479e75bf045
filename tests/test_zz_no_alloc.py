"""flint_moe_forward_noalloc: the layer forward for callers that cannot allocate
device memory at call time (runtimes that reserve all device memory up front,
hosts that forbid allocations on their serving path); its scratch is a fixed
array compiled into the library. Its output must match flint_moe_forward's,
which uses a caller workspace, and the oracle's, within the parity tolerance,
on two calls in a row (the second call runs on scratch that still holds the
first call's contents), across calls that switch weight type, batch size and
shape, and its device checks must reach flint_moe_noalloc_get_status.

This file is collected last so that a stop-at-first-failure run has already run
every other test."""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import synth
from gpu_layer import MAX_ABS_TOL_RMS, REL_L2_TOL, GpuLayer, bits_to_cuda, check_output, cuda_to_bits

pytestmark = pytest.mark.gpu

_LAYERS = {}


def _layer(name, wdtype="nvfp4"):
    base = "cfg0" if name == "cfg0" else "cfg1"
    key = (base, wdtype)
    if key not in _LAYERS:
        _LAYERS[key] = GpuLayer(synth.CONFIGS[base], seed=5, max_tokens=8, keep_f32=False, wdtype=wdtype)
    return _LAYERS[key]


def _close(a_bits, b_bits):
    a = synth.bf16_bits_to_f64(a_bits)
    b = synth.bf16_bits_to_f64(b_bits)
    rms = np.sqrt(np.mean(b ** 2))
    assert np.linalg.norm(a - b) <= REL_L2_TOL * np.linalg.norm(b)
    assert np.abs(a - b).max() <= MAX_ABS_TOL_RMS * rms


def _case(name, T, wdtype="nvfp4", seed=21):
    """One noalloc call checked against flint_moe_forward (caller workspace)
    and against the oracle on the ids the workspace call routed."""
    w = synth.CONFIGS[name]
    layer = _layer(name, wdtype)
    x_bits = synth.x_bits(seed, T, w.d)
    x = bits_to_cuda(x_bits)
    wr_bits = synth.make_router(w, seed, x_bits)
    wr = bits_to_cuda(wr_bits)
    res_bits = synth.x_bits(seed + 1, T, w.d)
    res = bits_to_cuda(res_bits)
    ref, ids, _ = layer.forward(x, wr, residual=res)
    out = torch.full_like(x, float("nan"))
    fm.flint_moe_forward_noalloc(x, T, wr, layer.weights, layer.shape, res, out)
    torch.cuda.synchronize()
    got = cuda_to_bits(out)
    _close(got, cuda_to_bits(ref))
    o = layer.oracle_forward(x_bits, wr_bits, ids.cpu().numpy(), residual_bits=res_bits)
    check_output(got, o["out"], f"noalloc {name} T={T} {wdtype}")


@pytest.mark.parametrize("name,T", [("cfg1", 1), ("cfg2", 8), ("cfg0", 4)])
def test_noalloc_matches_workspace_forward_twice(name, T):
    w = synth.CONFIGS[name]
    layer = _layer(name)
    x_bits = synth.x_bits(21, T, w.d)
    x = bits_to_cuda(x_bits)
    wr_bits = synth.make_router(w, 21, x_bits)
    wr = bits_to_cuda(wr_bits)
    res_bits = synth.x_bits(22, T, w.d)
    res = bits_to_cuda(res_bits)
    ref, ids, _ = layer.forward(x, wr, residual=res)
    outs = []
    for _ in range(2):
        out = torch.full_like(x, float("nan"))
        fm.flint_moe_forward_noalloc(x, T, wr, layer.weights, layer.shape, res, out)
        outs.append(out)
    torch.cuda.synchronize()
    ref_bits = cuda_to_bits(ref)
    o = layer.oracle_forward(x_bits, wr_bits, ids.cpu().numpy(), residual_bits=res_bits)
    for out in outs:
        _close(cuda_to_bits(out), ref_bits)
        check_output(cuda_to_bits(out), o["out"], f"noalloc {name} T={T}")
    rc, flags = fm.flint_moe_noalloc_get_status()
    assert rc == 0 and flags == 0


def test_noalloc_bf16_weights():
    # bf16 weights take the tensor-core path, which also fits the 1 MiB scratch
    _case("cfg1", 4, wdtype="bf16")


def test_noalloc_calls_switching_path_batch_and_shape():
    # NVFP4 batch 1 (single kernel), bf16 batch 4 (tensor-core path), NVFP4
    # batch 8, the reduced shape, then the Flint shape again at batch 1
    for i, (name, T, wd) in enumerate([("cfg1", 1, "nvfp4"), ("cfg1", 4, "bf16"), ("cfg2", 8, "nvfp4"),
                                       ("cfg0", 4, "nvfp4"), ("cfg1", 1, "nvfp4"), ("cfg1", 1, "nvfp4")]):
        _case(name, T, wdtype=wd, seed=40 + i)
    rc, flags = fm.flint_moe_noalloc_get_status()
    assert rc == 0 and flags == 0


def test_noalloc_status_reports_device_checks():
    # a bounded device wait that runs out, recorded in the built-in scratch's
    # status word, is reported once by flint_moe_noalloc_get_status
    scratch = fm.flint_debug_noalloc_scratch()
    assert scratch != 0
    fm.flint_debug_wait_timeout(scratch, 1000)
    rc, flags = fm.flint_moe_noalloc_get_status()
    assert rc == -7 and flags & 4
    rc, flags = fm.flint_moe_noalloc_get_status()
    assert rc == 0 and flags == 0
    _case("cfg1", 1, seed=60)  # the path still works afterwards


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
