"""Grouping by expert (row a3: expert histogram + token permutation) on the
GPU, bit-exact against the oracle's definition: each of the layer's three
grouping routines on random routings and on the extremes (every token on the
same experts; every selection on its own expert), a planted out-of-range id
reported as FLINT_DEVCHECK_EXPERT_ID, and whole-layer parity on routings
steered to those extremes."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import GpuLayer, bits_to_cuda, check_output, check_routing, cuda_to_bits

pytestmark = pytest.mark.gpu

MAX_T = {0: 128, 1: 10, 2: 32}  # tokens each routine takes at k = 6


def _ws(shape):
    ws = torch.empty(fm.flint_moe_workspace_bytes(shape, 1), dtype=torch.uint8, device="cuda")
    fm.flint_moe_workspace_init(ws)
    return ws


def _gpu_group(ids, E, S, impl):
    T, k = ids.shape
    shape = fm.Shape(2048, 512, E, k, S, fm.FLINT_W_NVFP4)
    ws = _ws(shape)
    d_ids = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()
    act = torch.full((E + S,), -7, dtype=torch.int32, device="cuda")
    off = torch.full((E + S + 1,), -7, dtype=torch.int32, device="cuda")
    pair = torch.full((T * (k + S),), -7, dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    fm.flint_debug_group(d_ids, T, shape, impl, act, off, pair, counts, ws)
    torch.cuda.synchronize()
    rc, flags = fm.flint_moe_get_status(ws)
    nr, na = counts.cpu().tolist()
    return act.cpu().numpy()[:na], off.cpu().numpy()[:na + 1], pair.cpu().numpy(), nr, rc, flags


def _expect_same(ids, E, S, impl):
    a, o, p, nr, rc, flags = _gpu_group(ids, E, S, impl)
    assert rc == 0 and flags == 0
    act, off, pair, nr_o = oracle.group(ids, E, S)
    assert nr == nr_o
    assert np.array_equal(a, act) and np.array_equal(o, off)
    assert np.array_equal(p[:off[-1]], pair)


@pytest.mark.parametrize("impl", [0, 1, 2])
def test_grouping_random_routings(impl):
    rng = np.random.default_rng(impl + 5)
    for T in sorted({1, 2, 3, 8, MAX_T[impl]}):
        if T > MAX_T[impl]:
            continue
        for E in (256, 40):
            ids = np.array([rng.choice(E, 6, replace=False) for _ in range(T)], np.int32)
            _expect_same(ids, E, 1, impl)
            _expect_same(ids, E, 0, impl)


@pytest.mark.parametrize("impl", [0, 1, 2])
def test_grouping_extremes(impl):
    T = MAX_T[impl]
    same = np.tile(np.array([200, 3, 77, 150, 9, 255], np.int32), (T, 1))
    _expect_same(same, 256, 1, impl)
    # every selection its own expert (T*6 <= 256 distinct ids, descending)
    Td = min(T, 256 // 6)
    distinct = np.arange(Td * 6, dtype=np.int32)[::-1].reshape(Td, 6).copy()
    _expect_same(distinct, 256, 1, impl)


@pytest.mark.parametrize("impl", [0, 1, 2])
def test_grouping_reports_out_of_range_ids(impl):
    ids = np.array([[1, 2, 300, 4, 5, 6], [7, 8, 9, 10, 11, -1]], np.int32)
    *_, rc, flags = _gpu_group(ids, 256, 1, impl)
    assert rc == -6 and flags & 1


def _layer_on_targets(layer, T, sets, seed, path=fm.FLINT_PATH_AUTO):
    w = layer.w
    x_bits = synth.x_bits(seed, T, w.d)
    wr_bits = synth.router_for_targets(w, seed, x_bits, sets)
    out, ids, gates = layer.forward(bits_to_cuda(x_bits), bits_to_cuda(wr_bits), path=path)
    torch.cuda.synchronize()
    ids_np = ids.cpu().numpy()
    assert sorted(map(tuple, np.sort(ids_np, axis=1).tolist())) == sorted(tuple(sorted(s)) for s in sets)
    check_routing(ids_np, gates.cpu().numpy(), oracle.router_logits(x_bits, wr_bits), w.k)
    ref = layer.oracle_forward(x_bits, wr_bits, ids_np)
    check_output(cuda_to_bits(out), ref["out"], f"T={T} steered routing")
    assert fm.flint_moe_get_status(layer.ws) == (0, 0)


@pytest.mark.parametrize("T", [8, 31, 128])
def test_layer_all_tokens_on_the_same_experts(T):
    # the largest single-expert token count each path can meet (T=128: the
    # tensor-core path's maximum)
    layer = GpuLayer(synth.CONFIGS["cfg1"], seed=17, max_tokens=T, keep_f32=False)
    _layer_on_targets(layer, T, [[200, 3, 77, 150, 9, 255]] * T, seed=300 + T)


@pytest.mark.parametrize("T", [8, 31, 42])
def test_layer_every_selection_on_its_own_expert(T):
    layer = GpuLayer(synth.CONFIGS["cfg1"], seed=18, max_tokens=T, keep_f32=False)
    sets = [list(range(6 * t, 6 * t + 6)) for t in range(T)]
    _layer_on_targets(layer, T, sets, seed=400 + T)
