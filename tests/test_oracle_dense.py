"""Pins of the oracle's dense NVFP4 matrix-vector product (the 4-bit output
head): closed forms on hand-built matrices (every code 1.0 at scale 1 gives the
sum of x; one-hot rows pick one element, scaled by the block scale and the
tensor scale; codes 8..15 negate), linearity in the tensor scale, row
selection, and agreement with the oracle's FFN building block on random data."""
import numpy as np
import pytest

import oracle
import synth


def _mat(codes, scales, ts):
    rows, half = codes.shape
    return oracle.NVFP4Matrix(np.ascontiguousarray(codes, np.uint8), np.ascontiguousarray(scales, np.uint8),
                              float(ts), rows, 2 * half)


def test_all_ones_rows_sum_x():
    rows, cols = 4, 64
    codes = np.full((rows, cols // 2), 0x22, np.uint8)   # both nibbles code 2 = 1.0
    scales = np.full((rows, cols // 16), 0x38, np.uint8)  # E4M3 0x38 = 1.0
    x = synth.x_bits(1, 3, cols)
    out = oracle.dense_gemv(_mat(codes, scales, 1.0), x)
    xs = synth.bf16_bits_to_f64(x).sum(axis=1)
    assert np.array_equal(out, np.repeat(xs[:, None], rows, axis=1))


def test_one_hot_rows_pick_elements():
    rows, cols = 6, 64
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.full((rows, cols // 16), 0x38, np.uint8)
    picks = [0, 1, 17, 30, 33, 63]
    vals = {0x1: 0.5, 0x7: 6.0, 0x9: -0.5, 0xF: -6.0, 0x3: 1.5, 0x5: 3.0}
    codev = list(vals)
    for r, c in enumerate(picks):
        codes[r, c // 2] = codev[r] << (4 * (c % 2))
    scales[3, picks[3] // 16] = 0x40  # 2.0
    x = synth.x_bits(2, 2, cols)
    out = oracle.dense_gemv(_mat(codes, scales, 0.25), x)
    xf = synth.bf16_bits_to_f64(x)
    for r, c in enumerate(picks):
        want = vals[codev[r]] * (2.0 if r == 3 else 1.0) * 0.25 * xf[:, c]
        assert np.array_equal(out[:, r], want)


def test_linear_in_tensor_scale_and_row_selection():
    rng = np.random.default_rng(4)
    w = rng.standard_normal((40, 128)).astype(np.float32) * 0.02
    m = oracle.quantize(w)
    x = synth.x_bits(4, 3, 128)
    full = oracle.dense_gemv(m, x)
    m2 = oracle.NVFP4Matrix(m.codes, m.scales, m.tensor_scale * 2.0, m.rows, m.cols)
    assert np.array_equal(oracle.dense_gemv(m2, x), 2.0 * full)
    rows = np.array([39, 0, 7, 7, 20], np.int32)
    assert np.array_equal(oracle.dense_gemv(m, x, rows), full[:, rows])
    with pytest.raises(ValueError):
        oracle.dense_gemv(m, x, np.array([40], np.int32))


def test_matches_decoded_matrix_product():
    rng = np.random.default_rng(5)
    w = rng.standard_normal((24, 256)).astype(np.float32) * 0.02
    m = oracle.quantize(w)
    x = synth.x_bits(5, 2, 256)
    np.testing.assert_allclose(oracle.dense_gemv(m, x), synth.bf16_bits_to_f64(x) @ oracle.decode(m).T,
                               rtol=1e-13, atol=1e-15)
