"""GPU packer and decoder parity: packed bytes, block scales and tensor scales
bit-exact against the oracle's quantiser and layout; decoded e2m1*e4m3
products bit-exact against the oracle's decode."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import GpuLayer

pytestmark = pytest.mark.gpu


def _oracle_pack(layer: GpuLayer, experts):
    trips = [layer.oracle_expert(e) for e in experts]
    return oracle.pack_layout(trips, layer.w.d, layer.w.inter)


def _expert_bytes(layer: GpuLayer, e):
    d, I = layer.w.d, layer.w.inter
    cpe, spe = 3 * I * d // 2, 3 * I * d // 16
    c = layer.packed[e * cpe:(e + 1) * cpe].cpu().numpy()
    s = layer.scales[e * spe:(e + 1) * spe].cpu().numpy()
    t = layer.tscales[3 * e:3 * e + 3].cpu().numpy()
    return c, s, t


def _assert_experts_equal(layer, experts):
    codes, scales, ts = _oracle_pack(layer, experts)
    d, I = layer.w.d, layer.w.inter
    cpe, spe = 3 * I * d // 2, 3 * I * d // 16
    for i, e in enumerate(experts):
        c, s, t = _expert_bytes(layer, e)
        np.testing.assert_array_equal(c, codes[i * cpe:(i + 1) * cpe], err_msg=f"codes of expert {e}")
        np.testing.assert_array_equal(s, scales[i * spe:(i + 1) * spe], err_msg=f"scales of expert {e}")
        np.testing.assert_array_equal(t.view(np.uint32), ts[3 * i:3 * i + 3].view(np.uint32))


def test_pack_cfg0_whole_layer_bit_exact():
    layer = GpuLayer(synth.CONFIGS["cfg0"], seed=0)
    _assert_experts_equal(layer, list(range(33)))


def test_pack_cfg1_sampled_experts_bit_exact():
    layer = GpuLayer(synth.CONFIGS["cfg1"], seed=0, max_tokens=1)
    _assert_experts_equal(layer, [0, 1, 97, 200, 255, 256])


def test_pack_edge_values_bit_exact():
    # crafted fp32 weights: exact ties of the E2M1 grid, saturation, signed
    # zeros, an all-zero expert, a zero block, tiny values, mixed magnitudes
    w = synth.CONFIGS["cfg0"]
    d, I, n = w.d, w.inter, w.E + w.S
    rng = np.random.default_rng(7)
    base = (rng.standard_normal((n, 3, I * d)) * 0.02).astype(np.float32)
    grid = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.5, 6.0, 4.5, -0.25, -2.5, -5.0, 0.0, -0.0, 1e-30],
                    np.float32)
    # expert 1 gate: blocks whose amax gives dec(sb)*s_t == 1 exactly -> ties land on the grid
    blk = np.tile(grid, I * d // 16)
    m = base[1, 0].copy()
    m[:] = blk
    m[0] = 2688.0  # tensor amax -> s_t = 1
    base[1, 0] = m
    base[2] = 0.0                       # all-zero expert
    base[3, 1, 32:48] = 0.0             # one zero block
    base[4, 2] *= np.float32(1e-20)     # tiny values
    base[5, 0, ::7] = -0.0
    base[6, 1, ::5] *= 1e4              # wide dynamic range in one tensor
    t = torch.from_numpy(base).cuda()
    layer = GpuLayer(w, weights_f32=t)
    _assert_experts_equal(layer, list(range(8)) + [32])


def test_pack_from_bf16_weights_bit_exact():
    w = synth.CONFIGS["cfg0"]
    d, I, n = w.d, w.inter, w.E + w.S
    wf = synth.layer_weights_torch(3, 0, n, d, I, 0.02)
    wb = wf.to(torch.bfloat16)
    shape = fm.Shape(d, I, w.E, w.k, w.S, 0)
    packed = torch.empty(fm.flint_packed_bytes(shape), dtype=torch.uint8, device="cuda")
    scales = torch.empty(fm.flint_block_scale_bytes(shape), dtype=torch.uint8, device="cuda")
    ts = torch.empty(n * 3, dtype=torch.float32, device="cuda")
    ws = torch.empty(fm.flint_moe_workspace_bytes(shape, 1), dtype=torch.uint8, device="cuda")
    fm.flint_pack_nvfp4(wb.view(torch.int16), 1, shape, packed, scales, ts, ws)
    # oracle quantises the same bf16 values (exact in fp32)
    layer_like = GpuLayer(w, weights_f32=wb.float())
    assert torch.equal(layer_like.packed, packed)
    assert torch.equal(layer_like.scales, scales)
    assert torch.equal(layer_like.tscales, ts)
    _assert_experts_equal(layer_like, [0, 11, 32])


def test_debug_dequant_products_bit_exact():
    layer = GpuLayer(synth.CONFIGS["cfg1"], seed=1, max_tokens=1)
    d, I = layer.w.d, layer.w.inter
    for e in (5, 256):
        g, u, dn = layer.oracle_expert(e)
        out = torch.empty((2 * 8, d), dtype=torch.float32, device="cuda")
        ts = fm.flint_debug_dequant(layer.weights, layer.shape, e, 0, 100, 8, out)
        got = out.cpu().numpy().astype(np.float64)
        for i in range(8):
            for which, m in ((0, g), (1, u)):
                want = oracle.decode(oracle.NVFP4Matrix(m.codes[100 + i:101 + i], m.scales[100 + i:101 + i], 1.0, 1, d))
                np.testing.assert_array_equal(got[2 * i + which], want[0])
        assert np.float32(ts[0]) == np.float32(g.tensor_scale) and np.float32(ts[1]) == np.float32(u.tensor_scale)
        out = torch.empty((16, I), dtype=torch.float32, device="cuda")
        ts = fm.flint_debug_dequant(layer.weights, layer.shape, e, 1, 2032, 16, out)
        want = oracle.decode(oracle.NVFP4Matrix(dn.codes[2032:], dn.scales[2032:], 1.0, 16, I))
        np.testing.assert_array_equal(out.cpu().numpy().astype(np.float64), want)
        assert np.float32(ts[0]) == np.float32(dn.tensor_scale)


def test_nonfinite_weight_flagged():
    w = synth.CONFIGS["cfg0"]
    d, I, n = w.d, w.inter, w.E + w.S
    wf = synth.layer_weights_torch(0, 0, n, d, I, 0.02)
    wf[3, 1, 77] = float("nan")
    shape = fm.Shape(d, I, w.E, w.k, w.S, 0)
    packed = torch.empty(fm.flint_packed_bytes(shape), dtype=torch.uint8, device="cuda")
    scales = torch.empty(fm.flint_block_scale_bytes(shape), dtype=torch.uint8, device="cuda")
    ts = torch.empty(n * 3, dtype=torch.float32, device="cuda")
    ws = torch.zeros(fm.flint_moe_workspace_bytes(shape, 1), dtype=torch.uint8, device="cuda")
    fm.flint_pack_nvfp4(wf, 0, shape, packed, scales, ts, ws)
    rc, flags = fm.flint_moe_get_status(ws)
    assert rc == -6 and flags & 2
    assert fm.flint_moe_get_status(ws) == (0, 0)  # reading clears it


def test_pack_bf16_layout():
    w = synth.CONFIGS["cfg0"]
    layer = GpuLayer(w, seed=2, wdtype="bf16")
    trips = [layer.oracle_expert(e) for e in range(w.E + w.S)]
    want = oracle.pack_layout_bf16(trips, w.d, w.inter)
    got = layer.packed.cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)
