"""Dequantised weights bit-exact, per decoder. The layer's tensor-core paths
decode NVFP4 with their own routines: the tcgen05 path writes e2m1 * e4m3 as
f16 into tensor memory (read back here with tcgen05.ld), the persistent
kernel's mma.sync variant builds the A fragments in registers (extracted here
through the MMA with one-hot B columns). Each decoded tile, times the fp32
tensor scale, must equal the oracle's fp64 decode exactly."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import GpuLayer

pytestmark = pytest.mark.gpu

_L = {}


def _layer():
    if "l" not in _L:
        _L["l"] = GpuLayer(synth.CONFIGS["cfg1"], seed=31, max_tokens=1)
    return _L["l"]


def _oracle_rows(layer, e, matrix):
    """fp64 decode of the packed rows of one expert matrix (gate/up rows interleaved)."""
    g, u, dn = layer.oracle_expert(e)
    if matrix == 1:
        return oracle.decode(dn)
    dg, du = oracle.decode(g), oracle.decode(u)
    out = np.empty((2 * dg.shape[0], dg.shape[1]))
    out[0::2], out[1::2] = dg, du
    return out


def _scale_rows(layer, e, matrix, rows):
    g, u, dn = layer.oracle_expert(e)
    if matrix == 1:
        return np.full(rows, dn.tensor_scale)
    return np.tile([g.tensor_scale, u.tensor_scale], rows // 2)


@pytest.mark.parametrize("decoder,matrix,row0,rows,k0,kn", [
    (0, 0, 0, 256, 0, 512), (0, 0, 768, 128, 1792, 256), (0, 1, 1920, 128, 256, 256),
    (1, 0, 0, 32, 0, 256), (1, 0, 1008, 16, 1920, 128), (1, 1, 0, 16, 0, 512), (1, 1, 2032, 16, 384, 128),
])
@pytest.mark.parametrize("expert", [3, 256])
def test_decoded_tiles_bit_exact(decoder, matrix, row0, rows, k0, kn, expert):
    layer = _layer()
    out = torch.full((rows, kn), float("nan"), dtype=torch.float32, device="cuda")
    fm.flint_debug_decode(layer.weights, layer.shape, expert, matrix, decoder, row0, rows, k0, kn, out)
    got = out.cpu().numpy().astype(np.float64)
    ref = _oracle_rows(layer, expert, matrix)[row0:row0 + rows, k0:k0 + kn]
    ts = _scale_rows(layer, expert, matrix, 2 * layer.w.inter if matrix == 0 else layer.w.d)[row0:row0 + rows]
    assert np.array_equal(got * ts[:, None], ref), np.argwhere(got * ts[:, None] != ref)[:5]


def test_decode_tiles_refuse_partial_tiles():
    layer = _layer()
    out = torch.empty((16, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(fm.FlintError):
        fm.flint_debug_decode(layer.weights, layer.shape, 0, 0, 0, 0, 16, 0, 128, out)  # tmem tiles are 128 x 256
    with pytest.raises(fm.FlintError):
        fm.flint_debug_decode(layer.weights, layer.shape, 0, 0, 1, 0, 8, 0, 128, out)  # fragment tiles are 16 rows
    with pytest.raises(fm.FlintError):
        fm.flint_debug_decode(layer.weights, layer.shape, 0, 0, 1, 0, 16, 64, 128, out)  # K tiles start at k0 % 128 == 0
