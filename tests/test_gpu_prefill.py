"""Prefill-size calls on the tensor-core path (more than 128 tokens): the
counting-sort grouping bit-exact against the oracle's definition, and the
layer against the fp64 oracle -- every token at a few hundred tokens (NVFP4
and bf16 weights, token counts that are not multiples of the 128-token
tiles), sampled tokens at 8192 tokens (the oracle computes any subset of
tokens: a token's output depends only on its own x and routing)."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import GpuLayer, bits_to_cuda, check_output, check_routing, cuda_to_bits

pytestmark = pytest.mark.gpu


def _group_large(ids, E, S):
    T, k = ids.shape
    shape = fm.Shape(2048, 512, E, k, S, fm.FLINT_W_NVFP4)
    ws = torch.empty(fm.flint_moe_workspace_bytes(shape, T), dtype=torch.uint8, device="cuda")
    fm.flint_moe_workspace_init(ws)
    d_ids = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()
    act = torch.full((E + S,), -7, dtype=torch.int32, device="cuda")
    off = torch.full((E + S + 1,), -7, dtype=torch.int32, device="cuda")
    pair = torch.full((T * (k + S),), -7, dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    fm.flint_debug_group(d_ids, T, shape, 3, act, off, pair, counts, ws)
    torch.cuda.synchronize()
    rc, flags = fm.flint_moe_get_status(ws)
    nr, na = counts.cpu().tolist()
    return act.cpu().numpy()[:na], off.cpu().numpy()[:na + 1], pair.cpu().numpy(), nr, rc, flags


@pytest.mark.parametrize("T,E,S", [(129, 256, 1), (300, 256, 1), (1000, 40, 1), (4096, 256, 1), (777, 13, 0),
                                   (64, 256, 1), (1, 8, 1)])
def test_large_t_grouping_matches_oracle(T, E, S):
    rng = np.random.default_rng(T + E)
    k = 6 if E >= 6 else E
    ids = np.array([rng.choice(E, k, replace=False) for _ in range(T)], np.int32)
    a, o, p, nr, rc, flags = _group_large(ids, E, S)
    assert rc == 0 and flags == 0
    act, off, pair, nr_o = oracle.group(ids, E, S)
    assert nr == nr_o
    assert np.array_equal(a, act) and np.array_equal(o, off)
    assert np.array_equal(p[:off[-1]], pair)


def test_large_t_grouping_extremes():
    rng = np.random.default_rng(3)
    T, E = 2048, 256
    # every token on the same six experts (each gets 2048 pairs: 16 token tiles)
    ids = np.tile(np.array([[5, 77, 3, 200, 128, 9]], np.int32), (T, 1))
    a, o, p, nr, rc, flags = _group_large(ids, E, 1)
    act, off, pair, nr_o = oracle.group(ids, E, 1)
    assert rc == 0 and nr == nr_o == 6
    assert np.array_equal(a, act) and np.array_equal(o, off) and np.array_equal(p[:off[-1]], pair)
    # a planted out-of-range id is skipped and reported
    ids = np.array([rng.choice(E, 6, replace=False) for _ in range(T)], np.int32)
    ids[1000, 2] = E + 3
    _, _, _, _, rc, flags = _group_large(ids, E, 1)
    assert rc == -6 and flags & 1  # status -6: a device check fired; flag 1: an expert id out of range


def _prefill_case(name, T, wdtype, seed, sample=None):
    w = synth.CONFIGS[name]
    layer = GpuLayer(w, seed=seed, max_tokens=T, keep_f32=False, wdtype=wdtype)
    x_bits = synth.x_bits(seed + 1, T, w.d)
    wr_bits = synth.to_bf16_bits(np.random.default_rng(seed).standard_normal((w.E, w.d)) * 0.02)
    x, wr = bits_to_cuda(x_bits), bits_to_cuda(wr_bits)
    out, ids, gates = layer.forward(x, wr)
    torch.cuda.synchronize()
    assert fm.flint_moe_get_status(layer.ws) == (0, 0)
    rows = np.arange(T) if sample is None else np.asarray(sample)
    ids_np, gates_np = ids.cpu().numpy()[rows], gates.cpu().numpy()[rows]
    check_routing(ids_np, gates_np, oracle.router_logits(x_bits[rows], wr_bits), w.k)
    ref = layer.oracle_forward(x_bits[rows], wr_bits, ids_np)
    check_output(cuda_to_bits(out)[rows], ref["out"], f"{name} T={T} {wdtype}")


@pytest.mark.parametrize("T", [129, 200, 333])
def test_prefill_nvfp4_every_token(T):
    _prefill_case("cfg1", T, "nvfp4", 40 + T)


def test_prefill_bf16_every_token():
    _prefill_case("cfg1", 257, "bf16", 41)


def test_prefill_8k_sampled_tokens():
    rng = np.random.default_rng(8)
    sample = np.sort(rng.choice(8192, 12, replace=False))
    _prefill_case("cfg1", 8192, "nvfp4", 42, sample=np.concatenate([[0, 127, 128, 8191], sample]))


def test_prefill_reduced_shape_every_token():
    # the reduced shape (d=512, inter=128 is below the NVFP4 tensor-core
    # minimum): bf16 weights at 500 tokens
    _prefill_case("cfg0", 500, "bf16", 43)
