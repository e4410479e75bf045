"""Expert-parallel layer pieces on one GPU against the oracle: the dispatch
kernel bit for bit against the oracle's plan (send order, local ids, gates,
source tokens, counts, pair positions, gathered rows; dropped ids), the
routed expert call against the oracle's layer output for the same routing,
and whole expert-parallel layer steps with 2, 4 and 8 ranks emulated in one
process (each phase run for every rank, the all-to-all replaced by copies
between the ranks' buffers, so no kernel ever waits on another) plus one rank
through NCCL's all-to-all, each rank's output against the oracle's layer
output. Bar: the layer contract's rel-L2 <= 5e-3; elementwise, the
contract's 2e-2 rms plus 2^-8 sum_j |g_j y_j| -- each of a token's expert rows
travels in bf16 (rounded once, 2^-9 relative, before the home rank sums
them), where the single-GPU layer rounds only the sum; the per-pair terms
g_j y_j come from the oracle's expert FFN."""
import dataclasses
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import nvfp4_weight_only_flint_b200 as fm
from nvfp4_weight_only_flint_b200 import ep
import oracle
import synth
from gpu_layer import GpuLayer, bits_to_cuda, check_output, cuda_to_bits

pytestmark = pytest.mark.gpu

FLINT = synth.CONFIGS["cfg4_nvfp4"]  # d 2048, I 512, 256 routed + 1 shared, top-6
SMALL = dataclasses.replace(FLINT, name="ep_small", d=512, inter=256, E=32, k=4, T=16)


def _dispatch(ids, gates, S, E, R, rank, x_bits):
    T, k = ids.shape
    d = x_bits.shape[1]
    P = T * (k + S)
    c = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).cuda()
    send_x = torch.full((max(P, 1), d), 0x7FC0, dtype=torch.int16, device="cuda")
    send_ids = torch.full((max(P, 1),), -7, dtype=torch.int32, device="cuda")
    send_gates = torch.zeros(max(P, 1), dtype=torch.float32, device="cuda")
    send_token = torch.full((max(P, 1),), -7, dtype=torch.int32, device="cuda")
    counts = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    pair_pos = torch.full((max(P, 1),), -9, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fm.flint_ep_dispatch(c(ids, np.int32), c(gates, np.float32), T, k, S, E, R, rank, c(x_bits, np.int16), d, send_x,
                         send_ids, send_gates, send_token, counts, pair_pos, status)
    torch.cuda.synchronize()
    n = int(counts.sum().item())
    return {"send_x": send_x[:n].cpu().numpy().view(np.uint16), "send_ids": send_ids[:n].cpu().numpy(),
            "send_gates": send_gates[:n].cpu().numpy(), "send_token": send_token[:n].cpu().numpy(),
            "counts": counts.cpu().numpy(), "pair_pos": pair_pos[:P].cpu().numpy().reshape(T, k + S),
            "status": int(status.item())}


@pytest.mark.parametrize("R,E,k,S,T", [(1, 256, 6, 1, 3), (2, 256, 6, 1, 64), (4, 256, 6, 1, 100),
                                       (8, 256, 6, 1, 2048), (8, 256, 8, 0, 5), (4, 32, 4, 1, 0)])
def test_dispatch_matches_oracle_plan(R, E, k, S, T):
    rng = np.random.default_rng(R * 1000 + T)
    ids = np.array([rng.choice(E, k, replace=False) for _ in range(T)], np.int32).reshape(T, k)
    gates = rng.random((T, k)).astype(np.float32)
    x = synth.to_bf16_bits(rng.standard_normal((max(T, 1), 512)).astype(np.float32))[:T]
    rank = R - 1
    got = _dispatch(ids, gates, S, E, R, rank, x)
    ref = oracle.ep_plan(ids, gates, S=S, E=E, R=R, rank=rank)
    for key in ("counts", "pair_pos", "send_ids", "send_gates", "send_token"):
        assert np.array_equal(got[key], ref[key]), key
    assert np.array_equal(got["send_x"], x[ref["send_token"]])
    assert got["status"] == 0


def test_dispatch_drops_out_of_range_ids():
    rng = np.random.default_rng(3)
    T, k, E, R = 10, 6, 256, 4
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    gates = rng.random((T, k)).astype(np.float32)
    ids[2, 1], ids[7, 5] = 256, -3
    x = synth.to_bf16_bits(rng.standard_normal((T, 512)).astype(np.float32))
    got = _dispatch(ids, gates, 1, E, R, 0, x)
    ref = oracle.ep_plan(ids, gates, S=1, E=E, R=R, rank=0)
    assert ref["dropped"] == 2
    assert got["status"] & fm.FLINT_DEVCHECK_EXPERT_ID
    for key in ("counts", "pair_pos", "send_ids", "send_gates", "send_token"):
        assert np.array_equal(got[key], ref[key]), key


_LAYERS = {}


def _layer(w, **kw):
    key = (w.name, tuple(sorted(kw.items())))
    if key not in _LAYERS:
        _LAYERS.clear()
        torch.cuda.empty_cache()
        _LAYERS[key] = GpuLayer(w, seed=0, **kw)
    return _LAYERS[key]


def _route(layer, x, wr, T):
    ids = torch.empty((T, layer.w.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((T, layer.w.k), dtype=torch.float32, device="cuda")
    fm.flint_moe_route(x, T, wr, layer.shape, ids, gates, layer.ws)
    return ids, gates


@pytest.mark.parametrize("T", [5, 64, 300])
def test_forward_routed_matches_oracle(T):
    w = FLINT
    layer = _layer(w, max_tokens=300, keep_f32=False)
    xb = synth.x_bits(400 + T, T, w.d)
    wrb = synth.make_router(w, 400 + T, xb)
    x, wr = bits_to_cuda(xb), bits_to_cuda(wrb)
    ids, gates = _route(layer, x, wr, T)
    out = torch.empty_like(x)
    fm.flint_moe_forward_routed(x, T, ids, gates, layer.weights, layer.shape, None, out, layer.ws)
    torch.cuda.synchronize()
    assert fm.flint_moe_get_status(layer.ws) == (0, 0)
    ref = layer.oracle_forward(xb, wrb, ids.cpu().numpy())
    check_output(cuda_to_bits(out), ref["out"], f"routed T={T}")


def _rank_layers(layer, R, wr, T):
    shape = layer.shape
    pshape = ep.packing_shape(shape, R)
    out = []
    for r in range(R):
        wl = ep.slice_rank_weights(layer.wf32, shape, r, R)
        packed = torch.empty(fm.flint_packed_bytes(pshape), dtype=torch.uint8, device="cuda")
        scales = torch.empty(fm.flint_block_scale_bytes(pshape), dtype=torch.uint8, device="cuda")
        tsc = torch.empty((pshape.n_experts + pshape.n_shared) * 3, dtype=torch.float32, device="cuda")
        fm.flint_pack_nvfp4(wl, 0, pshape, packed, scales, tsc, layer.ws)
        weights = fm.Weights(packed.data_ptr(), scales.data_ptr(), tsc.data_ptr())
        epl = ep.ExpertParallelLayer(shape, r, R, weights, wr, max_tokens=T)
        epl._keep = (packed, scales, tsc)
        out.append(epl)
    torch.cuda.synchronize()
    return out


def _emulated_step(layers, xs, T, residuals):
    """One layer step of R ranks in lockstep; the exchange is copies between
    the ranks' buffers in the order all_to_all_single delivers them."""
    R = len(layers)
    sc = [l.send(x, T).cpu().tolist() for l, x in zip(layers, xs)]  # sc[src][dst]
    for dst in range(R):
        n = 0
        for src in range(R):
            off, c = sum(sc[src][:dst]), sc[src][dst]
            s, l = layers[src], layers[dst]
            l.recv_x[n:n + c].copy_(s.send_x[off:off + c])
            l.recv_ids[n:n + c].copy_(s.send_ids[off:off + c])
            l.recv_gates[n:n + c].copy_(s.send_gates[off:off + c])
            n += c
        layers[dst].experts(n)
    outs = []
    for src in range(R):
        n = 0
        for dst in range(R):
            c = sc[src][dst]
            at = sum(sc[s2][dst] for s2 in range(src))  # where src's rows sit in dst's receive order
            layers[src].y_back[n:n + c].copy_(layers[dst].y[at:at + c])
            n += c
        out = torch.empty_like(xs[src])
        outs.append(layers[src].finish(T, out, residuals[src]))
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("w,R,T", [(SMALL, 2, 16), (SMALL, 4, 16), (SMALL, 8, 9), (FLINT, 8, 2)])
def test_ep_layer_emulated_ranks(w, R, T):
    layer = _layer(w, max_tokens=64, keep_f32=True)
    xbs = [synth.x_bits(500 + r, T, w.d) for r in range(R)]
    wrb = synth.make_router(w, 500, np.concatenate(xbs))
    wr = bits_to_cuda(wrb)
    resb = [synth.x_bits(600 + r, T, w.d) for r in range(R)] if w is SMALL else [None] * R
    layers = _rank_layers(layer, R, wr, T)
    outs = _emulated_step(layers, [bits_to_cuda(b) for b in xbs], T,
                          [bits_to_cuda(b) if b is not None else None for b in resb])
    for r in range(R):
        layers[r].check()  # raises on any device check flag of the step
        _check_ep(outs[r], layer, xbs[r], wrb, layers[r].ids[:T].cpu().numpy(), resb[r], f"rank {r} of {R}")


def _check_ep(out, layer, x_bits, wr_bits, ids, residual_bits, what):
    ref = layer.oracle_forward(x_bits, wr_bits, ids, residual_bits=residual_bits)
    w = layer.w
    x = synth.bf16_bits_to_f64(x_bits)
    mag = np.zeros_like(ref["out"])
    for t in range(x.shape[0]):
        for j in range(w.k):
            mag[t] += np.abs(ref["gates"][t, j] * oracle.expert_ffn(layer.oracle_expert(int(ids[t, j])), x[t]))
        for s in range(w.S):
            mag[t] += np.abs(oracle.expert_ffn(layer.oracle_expert(w.E + s), x[t]))
    got = synth.bf16_bits_to_f64(cuda_to_bits(out))
    ref_out = ref["out"]
    rel = np.linalg.norm(got - ref_out) / np.linalg.norm(ref_out)
    assert rel <= 5e-3, f"{what}: rel L2 {rel:.3e}"
    rms = np.sqrt(np.mean(ref_out ** 2))
    tol = 2e-2 * rms + 2.0 ** -8 * mag
    bad = np.abs(got - ref_out) > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst excess {np.max(np.abs(got - ref_out) - tol):.3e}"


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ep_layer_one_rank_through_nccl():
    w, T = SMALL, 16
    layer = _layer(w, max_tokens=64, keep_f32=True)
    xb = synth.x_bits(700, T, w.d)
    wrb = synth.make_router(w, 700, xb)
    wr = bits_to_cuda(wrb)
    torch.cuda.set_device(0)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        (epl,) = _rank_layers(layer, 1, wr, T)
        x = bits_to_cuda(xb)
        out = torch.empty_like(x)
        epl.forward(x, T, out, exchange=ep.AllToAll())
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    _check_ep(out, layer, xb, wrb, epl.ids[:T].cpu().numpy(), None, "one rank, NCCL all-to-all")
