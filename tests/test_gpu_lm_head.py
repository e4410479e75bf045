"""The 4-bit output head (dense NVFP4 GEMV, 150,144 x 2048 at the Flint shape)
against the oracle: packed planes bit-exact with the oracle's quantiser, and
logits within rel L2 <= 5e-3, max-abs <= 2e-2 * rms on all rows of a small
head and on sampled rows (plus the first and last) of the full-size head,
at one, two and eight tokens; shape edges (rows not a multiple of the 16-row
tile, one row); wide-range x."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth
from gpu_layer import bits_to_cuda

pytestmark = pytest.mark.gpu

VOCAB = 150144


def _ws():
    ws = torch.zeros(2048, dtype=torch.uint8, device="cuda")
    return ws


def _pack(w_f32_cuda, rows, cols, ws):
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device="cuda")
    ts = torch.empty(4, dtype=torch.float32, device="cuda")
    fm.flint_pack_nvfp4_dense(w_f32_cuda, 0, rows, cols, codes, scales, ts, ws)
    return codes, scales, ts


def _run(codes, scales, ts, x_bits, rows, cols, ws):
    T = x_bits.shape[0]
    out = torch.full((T, rows), float("nan"), dtype=torch.float32, device="cuda")
    fm.flint_lm_head(bits_to_cuda(x_bits), T, codes, scales, ts, rows, cols, out, ws)
    torch.cuda.synchronize()
    assert fm.flint_moe_get_status(ws) == (0, 0)
    return out.cpu().numpy().astype(np.float64)


def _check(got, ref, what):
    for t in range(ref.shape[0]):
        d = got[t] - ref[t]
        assert np.linalg.norm(d) <= 5e-3 * np.linalg.norm(ref[t]), what
        assert np.abs(d).max() <= 2e-2 * np.sqrt(np.mean(ref[t] ** 2)), what


@pytest.mark.parametrize("rows,cols,T", [(1, 512, 1), (37, 512, 2), (5000, 1024, 8), (2367, 2048, 1),
                                         (2367, 2048, 5), (300, 4096, 1), (300, 4096, 8)])
def test_small_heads_all_rows(rows, cols, T):
    ws = _ws()
    rng = np.random.default_rng(rows + cols)
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    codes, scales, ts = _pack(torch.from_numpy(w).cuda(), rows, cols, ws)
    m = oracle.quantize(w)
    assert np.array_equal(codes.cpu().numpy(), m.codes) and np.array_equal(scales.cpu().numpy(), m.scales)
    assert ts[0].item() == np.float32(m.tensor_scale)
    x = synth.x_bits(rows, T, cols)
    _check(_run(codes, scales, ts, x, rows, cols, ws), oracle.dense_gemv(m, x), f"{rows}x{cols} T={T}")


@pytest.mark.parametrize("T", [1, 2, 8])
def test_flint_head_sampled_rows(T):
    rows, cols = VOCAB, 2048
    ws = _ws()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(synth.key(7, "experts", 999) & 0x7FFFFFFFFFFFFFFF)
    w = torch.randn((rows, cols), generator=gen, device="cuda", dtype=torch.float32).mul_(0.02)
    codes, scales, ts = _pack(w, rows, cols, ws)
    x = synth.x_bits(77, T, cols)
    got = _run(codes, scales, ts, x, rows, cols, ws)
    sample = np.unique(np.concatenate([np.random.default_rng(T).choice(rows, 3000, replace=False),
                                       [0, 1, 15, 16, rows - 17, rows - 1]])).astype(np.int32)
    # the oracle quantises the sampled rows itself from the same fp32 draws
    # (the tensor scale comes from the whole matrix's amax, a plain max)
    wa = w[torch.from_numpy(sample).cuda().long()].cpu().numpy()
    amax = float(np.abs(w.cpu().numpy()).max())  # over the whole matrix, on the host
    m = oracle.quantize_with_tensor_scale(wa, amax)
    assert np.array_equal(codes[torch.from_numpy(sample).cuda().long()].cpu().numpy(), m.codes)
    _check(got[:, sample], oracle.dense_gemv(m, x), f"head T={T}")


def test_head_wide_range_x():
    rows, cols = 4096, 2048
    ws = _ws()
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    codes, scales, ts = _pack(torch.from_numpy(w).cuda(), rows, cols, ws)
    xf = rng.standard_normal((2, cols)).astype(np.float32)
    xf[0, :5] = [1e3, -1e3, 1e-4, 6e4, -3e-5]
    xf[1] *= 1e-3
    x = synth.to_bf16_bits(xf)
    _check(_run(codes, scales, ts, x, rows, cols, ws), oracle.dense_gemv(oracle.quantize(w), x), "wide x")


def test_head_rejects_bad_shapes():
    ws = _ws()
    z = torch.zeros(64, dtype=torch.uint8, device="cuda")
    f = torch.zeros(64, dtype=torch.float32, device="cuda")
    x = torch.zeros((9, 2048), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fm.FlintError):
        fm.flint_lm_head(x, 9, z, z, f, 16, 2048, f, ws)   # nine tokens
    with pytest.raises(fm.FlintError):
        fm.flint_lm_head(x, 1, z, z, f, 16, 1000, f, ws)   # cols not supported
