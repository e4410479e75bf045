"""GPU router parity: routed ids bit-exact against the oracle (tokens whose
6th/7th softmax gap is below 1e-6 are reported, not compared), gates within
fp32 rounding, for the layer workloads and ragged token counts."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import bits_to_cuda, check_routing

pytestmark = pytest.mark.gpu


def _route(x_bits, wr_bits, E, k, d):
    T = x_bits.shape[0]
    shape = fm.Shape(d, 512 if d >= 2048 else 128, E, k, 1, 0)
    ws = torch.empty(fm.flint_moe_workspace_bytes(shape, T), dtype=torch.uint8, device="cuda")
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gates = torch.empty((T, k), dtype=torch.float32, device="cuda")
    fm.flint_moe_route(bits_to_cuda(x_bits), T, bits_to_cuda(wr_bits), shape, ids, gates, ws)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), gates.cpu().numpy()


@pytest.mark.parametrize("name", ["cfg0", "cfg1", "cfg2", "cfg4_nvfp4"])
def test_route_workloads(name):
    w = synth.CONFIGS[name]
    x = synth.x_bits(0, w.T, w.d)
    wr = synth.make_router(w, 0, x)
    ids, gates = _route(x, wr, w.E, w.k, w.d)
    near = check_routing(ids, gates, oracle.router_logits(x, wr), w.k)
    assert len(near) <= max(1, w.T // 16), near
    if name == "cfg2":
        frac = synth.overlap_fraction(ids)
        assert 0.3 <= frac <= 0.5, frac


@pytest.mark.parametrize("T", [1, 2, 3, 7, 9, 17, 31, 32, 100, 1000])
def test_route_ragged_token_counts(T):
    w = synth.CONFIGS["cfg1"]
    x = synth.x_bits(T, T, w.d)
    wr = synth.make_router(w, 1, x)
    ids, gates = _route(x, wr, w.E, w.k, w.d)
    check_routing(ids, gates, oracle.router_logits(x, wr), w.k)


def test_route_all_equal_logits_lowest_indices():
    x = synth.x_bits(0, 5, 2048)
    wr = np.zeros((256, 2048), np.uint16)
    ids, gates = _route(x, wr, 256, 6, 2048)
    assert ids.tolist() == [[0, 1, 2, 3, 4, 5]] * 5
    np.testing.assert_allclose(gates, 1 / 6, rtol=0, atol=1e-7)


def test_route_single_expert():
    x = synth.x_bits(4, 3, 512)
    wr = synth.to_bf16_bits(np.random.default_rng(0).standard_normal((1, 512)) * 0.02)
    ids, gates = _route(x, wr, 1, 1, 512)
    assert ids.tolist() == [[0]] * 3 and gates.tolist() == [[1.0]] * 3


def test_route_k_eight_of_512():
    x = synth.x_bits(9, 6, 1024)
    wr = synth.to_bf16_bits(np.random.default_rng(9).standard_normal((512, 1024)) * 0.02)
    T = 6
    shape = fm.Shape(1024, 256, 512, 8, 0, 0)
    ws = torch.empty(fm.flint_moe_workspace_bytes(shape, T), dtype=torch.uint8, device="cuda")
    ids = torch.empty((T, 8), dtype=torch.int32, device="cuda")
    gates = torch.empty((T, 8), dtype=torch.float32, device="cuda")
    fm.flint_moe_route(bits_to_cuda(x), T, bits_to_cuda(wr), shape, ids, gates, ws)
    check_routing(ids.cpu().numpy(), gates.cpu().numpy(), oracle.router_logits(x, wr), 8)
