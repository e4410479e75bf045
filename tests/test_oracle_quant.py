"""Pins of the oracle's NVFP4 quantiser (the fp32 recipe).

Recipe: s_t = amax/2688 (1 if amax = 0); per 16-element block along K
sb = E4M3((amax_b/6)/s_t); q = E2M1(w/(dec(sb)*s_t)); q = 0 when dec(sb) = 0.
"""
import numpy as np
import pytest

import oracle


def _dec(m):
    return oracle.decode(m)


def test_round_trip_every_code_with_exact_scales():
    # A tensor whose amax is 2688 has s_t = 1 exactly; a block whose amax is
    # 6*dec(sb) then reproduces sb exactly, and every code value * dec(sb)
    # reproduces its code.
    rng = np.random.default_rng(0)
    sbs = [0x7E, 0x38, 0x40, 0x20, 0x08, 0x10, 0x3A, 0x55]
    rows = []
    codes_want = []
    for sb in sbs:
        s = oracle.e4m3_decode(sb)
        for _ in range(4):
            c = rng.integers(0, 16, size=16)
            c[rng.integers(16)] = 0x7  # the block max: 6*s
            rows.append([oracle.e2m1_decode(int(ci)) * s for ci in c])
            codes_want.append(c)
    w = np.array(rows, dtype=np.float32).reshape(len(sbs) * 4, 16)
    m = oracle.quantize(w)
    assert m.tensor_scale == 1.0
    for r in range(w.shape[0]):
        assert m.scales[r, 0] == sbs[r // 4]
        got = [(m.codes[r, j // 2] >> (4 * (j % 2))) & 0xF for j in range(16)]
        want = codes_want[r]
        for g, wv, val in zip(got, want, w[r]):
            # -0.0 (code 8) and +0.0 (code 0) both reproduce a zero value
            if val == 0.0:
                assert g in (0, 8)
            else:
                assert g == wv
    np.testing.assert_array_equal(_dec(m), w.astype(np.float64))


def test_zero_tensor_and_zero_block():
    m = oracle.quantize(np.zeros((4, 32), np.float32))
    assert m.tensor_scale == 1.0
    assert not m.codes.any() and not m.scales.any()
    w = np.zeros((2, 32), np.float32)
    w[0, 16:] = np.linspace(-1, 1, 16)
    m = oracle.quantize(w)
    assert m.scales[0, 0] == 0 and m.scales[1, 0] == 0 and m.scales[1, 1] == 0
    assert m.codes[0, :8].tolist() == [0] * 8


def test_tensor_scale_and_block_scale_values():
    w = np.zeros((1, 32), np.float32)
    w[0, 3] = 5.376  # tensor amax -> s_t = 5.376/2688 = 0.002 (fp32)
    w[0, 20] = -0.1
    m = oracle.quantize(w)
    st = np.float32(np.float32(5.376) / np.float32(2688.0))
    assert m.tensor_scale == float(st)
    # block 1: (0.1/6)/s_t = 8.333.. -> E4M3 8.0 (0x50); q = -0.1/(8*s_t) = -6.25 -> saturates to -6
    v = np.float32(np.float32(np.float32(0.1) / np.float32(6.0)) / st)
    assert oracle.e4m3_encode(float(v)) == m.scales[0, 1]
    assert oracle.e4m3_decode(int(m.scales[0, 1])) == 8.0
    assert (m.codes[0, 10] & 0xF) == 0xF


def test_quantisation_error_bound():
    # every element lands on the nearest representable value of its block grid,
    # so |w - deq| <= half the largest grid step, (6-4)/2 * dec(sb) * s_t,
    # plus the block scale rounding headroom (|w| may exceed 6*dec(sb)*s_t by
    # the E4M3 rounding of (amax_b/6)/s_t, at most 1/16 relative)
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    m = oracle.quantize(w)
    deq = _dec(m)
    for r in range(64):
        for b in range(16):
            s = oracle.e4m3_decode(int(m.scales[r, b])) * m.tensor_scale
            blk = w[r, 16 * b:16 * b + 16].astype(np.float64)
            err = np.abs(blk - deq[r, 16 * b:16 * b + 16])
            assert err.max() <= 1.0 * s + np.abs(blk).max() / 16 + 1e-12


def test_quantiser_picks_nearest_code_brute_force():
    # For each element, the chosen code is the nearest of the 16 codes on the
    # grid dec(code) * dec(sb) * s_t to w/(dec(sb)*s_t) (fp32 quotient), ties
    # to the even code: exhaustive search over the codes.
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((8, 64)) * 0.03).astype(np.float32)
    m = oracle.quantize(w)
    st = np.float32(m.tensor_scale)
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for r in range(8):
        for c in range(64):
            sb = int(m.scales[r, c // 16])
            denom = np.float32(np.float32(oracle.e4m3_decode(sb)) * st)
            qv = float(np.float32(w[r, c] / denom))
            a = min(abs(qv), 6.0)
            best = min(range(8), key=lambda i: (abs(a - mags[i]), i % 2))
            code = (m.codes[r, c // 2] >> (4 * (c % 2))) & 0xF
            assert code & 7 == best
            assert (code >> 3) == (1 if qv < 0 or (qv == 0 and np.signbit(qv)) else 0)


def test_rejects_non_finite():
    w = np.zeros((1, 16), np.float32)
    w[0, 5] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(w)


def test_rows_of_a_larger_tensor_match_the_whole():
    # quantising a subset of rows with the whole tensor's amax gives exactly
    # those rows of the whole tensor's quantisation
    rng = np.random.default_rng(21)
    w = (rng.standard_normal((50, 64)) * 0.02).astype(np.float32)
    whole = oracle.quantize(w)
    rows = [3, 0, 49, 17]
    part = oracle.quantize_with_tensor_scale(w[rows], float(np.abs(w).max()))
    assert part.tensor_scale == whole.tensor_scale
    assert np.array_equal(part.codes, whole.codes[rows]) and np.array_equal(part.scales, whole.scales[rows])
    with pytest.raises(ValueError):  # a value above the stated amax
        oracle.quantize_with_tensor_scale(w[rows], float(np.abs(w[rows]).max()) / 2)
