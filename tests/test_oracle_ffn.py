"""Pins of the oracle's experts and layer: reductions to a dense SwiGLU FFN
(numpy matmuls on the decoded weights), all-experts softmax mixture, zero
input, linearity in the down tensor scale, and the packed layout."""
import numpy as np
import pytest

import oracle
import synth


def _dense_swiglu(trip, x):
    """Dense SwiGLU with numpy: W_d (silu(W_g x) * (W_u x)) on decoded weights."""
    g, u, dn = (oracle.decode(m) for m in trip)
    a, b = g @ x, u @ x
    return dn @ (a / (1.0 + np.exp(-a)) * b)


def _experts(n, d, inter, seed=0, layer=0):
    out = []
    for e in range(n):
        g, u, dn = synth.expert_weights_np(seed, layer, e, d, inter)
        out.append((oracle.quantize(g), oracle.quantize(u), oracle.quantize(dn)))
    return out


def test_single_expert_layer_equals_dense_ffn():
    d, inter = 64, 32
    ex = _experts(1, d, inter)
    x = synth.x_bits(0, 3, d)
    wr = synth.to_bf16_bits(np.random.default_rng(0).standard_normal((1, d)) * 0.02)
    r = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=1, k=1, S=0)
    xf = synth.bf16_bits_to_f64(x)
    for t in range(3):
        np.testing.assert_allclose(r["out"][t], _dense_swiglu(ex[0], xf[t]), rtol=1e-12, atol=1e-14)
    assert np.all(r["gates"] == 1.0) and np.all(r["ids"] == 0)


def test_expert_ffn_equals_dense():
    d, inter = 128, 64
    ex = _experts(1, d, inter, seed=3)
    xf = synth.bf16_bits_to_f64(synth.x_bits(3, 1, d))[0]
    np.testing.assert_allclose(oracle.expert_ffn(ex[0], xf), _dense_swiglu(ex[0], xf), rtol=1e-12, atol=1e-14)


def test_all_experts_is_softmax_mixture_plus_shared():
    d, inter, E = 64, 32, 5
    ex = _experts(E + 1, d, inter, seed=1)
    x = synth.x_bits(1, 2, d)
    wr = synth.to_bf16_bits(np.random.default_rng(1).standard_normal((E, d)) * 0.3)
    r = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=E, k=E, S=1)
    xf = synth.bf16_bits_to_f64(x)
    wrf = synth.bf16_bits_to_f64(wr)
    for t in range(2):
        l = wrf @ xf[t]
        p = np.exp(l - l.max())
        p /= p.sum()
        want = sum(p[e] * _dense_swiglu(ex[e], xf[t]) for e in range(E)) + _dense_swiglu(ex[E], xf[t])
        np.testing.assert_allclose(r["out"][t], want, rtol=1e-11, atol=1e-13)


def test_zero_input_zero_output():
    d, inter, E = 64, 32, 8
    ex = _experts(E + 1, d, inter, seed=2)
    x = np.zeros((2, d), np.uint16)
    wr = synth.to_bf16_bits(np.random.default_rng(2).standard_normal((E, d)) * 0.02)
    r = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=E, k=6, S=1)
    assert not r["out"].any()
    assert r["ids"].tolist() == [[0, 1, 2, 3, 4, 5]] * 2


def test_residual_is_added():
    d, inter, E = 64, 32, 8
    ex = _experts(E + 1, d, inter, seed=2)
    x = synth.x_bits(5, 2, d)
    res = synth.x_bits(6, 2, d)
    wr = synth.to_bf16_bits(np.random.default_rng(2).standard_normal((E, d)) * 0.02)
    a = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=E, k=6, S=1)["out"]
    b = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=E, k=6, S=1, residual_bits=res)["out"]
    np.testing.assert_allclose(b - a, synth.bf16_bits_to_f64(res), rtol=0, atol=1e-12)


def test_linear_in_down_tensor_scale():
    d, inter, E = 64, 32, 8
    ex = _experts(E + 1, d, inter, seed=4)
    x = synth.x_bits(4, 1, d)
    wr = synth.to_bf16_bits(np.random.default_rng(4).standard_normal((E, d)) * 0.02)
    base = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=E, k=6, S=1)
    e = int(base["ids"][0, 2])
    g, u, dn = ex[e]
    dn2 = oracle.NVFP4Matrix(dn.codes, dn.scales, dn.tensor_scale * 2.0, dn.rows, dn.cols)
    ex2 = list(ex)
    ex2[e] = (g, u, dn2)
    two = oracle.moe_forward(x, wr, ex2, d=d, inter=inter, E=E, k=6, S=1)
    contrib = base["gates"][0, 2] * oracle.expert_ffn(ex[e], synth.bf16_bits_to_f64(x)[0])
    np.testing.assert_allclose(two["out"][0] - base["out"][0], contrib, rtol=1e-10, atol=1e-14)


def test_forced_ids_renormalise_their_probabilities():
    d, inter, E = 64, 32, 8
    ex = _experts(E + 1, d, inter, seed=5)
    x = synth.x_bits(7, 1, d)
    wr = synth.to_bf16_bits(np.random.default_rng(5).standard_normal((E, d)) * 0.1)
    forced = np.array([[7, 0, 3]], np.int32)
    r = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=E, k=3, S=0, ids_override=forced)
    l = r["logits"][0]
    p = np.exp(l[[7, 0, 3]] - l.max())
    np.testing.assert_allclose(r["gates"][0], p / p.sum(), rtol=1e-14)
    xf = synth.bf16_bits_to_f64(x)[0]
    want = sum(r["gates"][0, j] * _dense_swiglu(ex[e], xf) for j, e in enumerate([7, 0, 3]))
    np.testing.assert_allclose(r["out"][0], want, rtol=1e-11, atol=1e-14)


def test_threads_do_not_change_results():
    d, inter, E = 64, 32, 16
    ex = _experts(E + 1, d, inter, seed=6)
    x = synth.x_bits(8, 5, d)
    wr = synth.to_bf16_bits(np.random.default_rng(6).standard_normal((E, d)) * 0.05)
    a = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=E, k=6, S=1, n_threads=1)["out"]
    b = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=E, k=6, S=1, n_threads=4)["out"]
    assert np.array_equal(a, b)


def test_packed_layout_offsets():
    # d=32, I=32, two experts: check where individual bytes land
    d, inter = 32, 32
    ex = []
    for e in range(2):
        trip = []
        for m in range(3):
            rows, cols = (inter, d) if m < 2 else (d, inter)
            codes = (np.arange(rows * cols // 2, dtype=np.int64) * 7 + 31 * e + 101 * m).astype(np.uint8).reshape(rows, cols // 2)
            scales = (np.arange(rows * cols // 16, dtype=np.int64) * 3 + 17 * e + 53 * m).astype(np.uint8).reshape(rows, cols // 16)
            trip.append(oracle.NVFP4Matrix(codes, scales, 1.0 + e + 0.25 * m, rows, cols))
        ex.append(tuple(trip))
    codes, scales, ts = oracle.pack_layout(ex, d, inter)
    cpe, spe = 3 * inter * d // 2, 3 * inter * d // 16
    assert codes.size == 2 * cpe and scales.size == 2 * spe
    for e in range(2):
        g, u, dn = ex[e]
        for i in (0, 5, 31):
            assert codes[e * cpe + i * d + 3] == g.codes[i, 3]
            assert codes[e * cpe + i * d + d // 2 + 3] == u.codes[i, 3]
            assert scales[e * spe + i * d // 8 + 1] == g.scales[i, 1]
            assert scales[e * spe + i * d // 8 + d // 16 + 1] == u.scales[i, 1]
        for n in (0, 9, 31):
            assert codes[e * cpe + inter * d + n * inter // 2 + 15] == dn.codes[n, 15]
            assert scales[e * spe + inter * d // 8 + n * inter // 16 + 1] == dn.scales[n, 1]
        assert ts[3 * e: 3 * e + 3].tolist() == [1.0 + e, 1.25 + e, 1.5 + e]


def test_input_norm_single_expert_equals_dense_on_normalised_x():
    # weightless RMS normalisation of the layer input: xn = x / sqrt(mean(x^2) + 1e-6)
    d, inter = 64, 32
    ex = _experts(1, d, inter, seed=9)
    x = synth.x_bits(9, 3, d)
    res = synth.x_bits(10, 3, d)
    wr = synth.to_bf16_bits(np.random.default_rng(9).standard_normal((1, d)) * 0.02)
    r = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=1, k=1, S=0, residual_bits=res, input_norm=True)
    xf = synth.bf16_bits_to_f64(x)
    for t in range(3):
        xn = xf[t] / np.sqrt(np.mean(xf[t] ** 2) + 1e-6)
        want = _dense_swiglu(ex[0], xn) + synth.bf16_bits_to_f64(res)[t]
        np.testing.assert_allclose(r["out"][t], want, rtol=1e-12, atol=1e-13)


def test_input_norm_router_sees_normalised_x():
    d, E = 64, 8
    x = synth.x_bits(11, 2, d)
    wr = synth.to_bf16_bits(np.random.default_rng(11).standard_normal((E, d)) * 0.3)
    ex = _experts(E, d, 32, seed=11)
    r = oracle.moe_forward(x, wr, ex, d=d, inter=32, E=E, k=2, S=0, input_norm=True)
    xf = synth.bf16_bits_to_f64(x)
    rms = np.sqrt(np.mean(xf ** 2, axis=1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(r["logits"], (xf / rms) @ synth.bf16_bits_to_f64(wr).T, rtol=1e-12)


# ---------------------------------------------------------------- bf16 weights
def _np_bf16(bits):
    """bf16 bit patterns -> fp64 by widening the pattern to an fp32 one (numpy
    only, independent of the oracle's decoder)."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _bf16_experts(n, d, inter, seed=0, layer=0):
    out = []
    for e in range(n):
        g, u, dn = synth.expert_weights_np(seed, layer, e, d, inter)
        out.append(tuple(oracle.BF16Matrix(synth.to_bf16_bits(m), m.shape[0], m.shape[1]) for m in (g, u, dn)))
    return out


def _np_dense_swiglu_bf16(trip, x):
    g, u, dn = (_np_bf16(m.bits) for m in trip)
    a, b = g @ x, u @ x
    return dn @ (a / (1.0 + np.exp(-a)) * b)


def test_bf16_decode_is_exact_widening():
    # +0, -0, smallest subnormal, a subnormal, 1, -1.5, largest finite, 2^-126,
    # 3.140625 (0x4049), -65280 (0xC77F)
    bits = np.array([[0x0000, 0x8000, 0x0001, 0x0050, 0x3F80],
                     [0xBFC0, 0x7F7F, 0x0080, 0x4049, 0xC77F]], np.uint16)
    got = oracle.decode(oracle.BF16Matrix(bits, 2, 5))
    want = np.array([[0.0, -0.0, 2.0 ** -133, 80 * 2.0 ** -133, 1.0],
                     [-1.5, (2 - 2 ** -7) * 2.0 ** 127, 2.0 ** -126, 3.140625, -65280.0]])
    assert np.array_equal(got, want)
    assert np.signbit(got[0, 1])
    # random patterns of finite values: the decode is the fp32 widening
    rng = np.random.default_rng(3)
    r = rng.integers(0, 1 << 16, size=(16, 32), dtype=np.uint32).astype(np.uint16)
    r[(r & 0x7F80) == 0x7F80] = 0x3F80  # no inf/NaN patterns
    assert np.array_equal(oracle.decode(oracle.BF16Matrix(r, 16, 32)), _np_bf16(r))


def test_bf16_single_expert_layer_equals_dense_ffn():
    d, inter = 64, 32
    ex = _bf16_experts(1, d, inter, seed=12)
    x = synth.x_bits(12, 3, d)
    wr = synth.to_bf16_bits(np.random.default_rng(12).standard_normal((1, d)) * 0.02)
    r = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=1, k=1, S=0)
    xf = _np_bf16(x)
    for t in range(3):
        np.testing.assert_allclose(r["out"][t], _np_dense_swiglu_bf16(ex[0], xf[t]), rtol=1e-12, atol=1e-14)


def test_bf16_layer_is_renormalised_mixture_plus_shared():
    d, inter, E, k = 64, 32, 6, 2
    ex = _bf16_experts(E + 1, d, inter, seed=13)
    x = synth.x_bits(13, 2, d)
    wr = synth.to_bf16_bits(np.random.default_rng(13).standard_normal((E, d)) * 0.3)
    r = oracle.moe_forward(x, wr, ex, d=d, inter=inter, E=E, k=k, S=1)
    xf, wrf = _np_bf16(x), _np_bf16(wr)
    for t in range(2):
        l = wrf @ xf[t]
        sel = sorted(range(E), key=lambda e: (-l[e], e))[:k]
        p = np.exp(l[sel] - l.max())
        p /= p.sum()
        want = sum(p[j] * _np_dense_swiglu_bf16(ex[e], xf[t]) for j, e in enumerate(sel))
        want = want + _np_dense_swiglu_bf16(ex[E], xf[t])
        assert r["ids"][t].tolist() == sel
        np.testing.assert_allclose(r["out"][t], want, rtol=1e-11, atol=1e-13)


def test_packed_layout_bf16_offsets():
    # d=32, I=32, two experts, every element a distinct pattern: unit u of
    # expert e = [gate row u | up row u] at element e*3*I*d + u*2d; down row n
    # at e*3*I*d + 2*I*d + n*I
    d, inter = 32, 32
    ex = []
    for e in range(2):
        trip = []
        for m in range(3):
            rows, cols = (inter, d) if m < 2 else (d, inter)
            bits = ((np.arange(rows * cols, dtype=np.int64) * 3 + 4096 * m + 12288 * e) % 65536).astype(np.uint16)
            trip.append(oracle.BF16Matrix(bits.reshape(rows, cols), rows, cols))
        ex.append(tuple(trip))
    out = oracle.pack_layout_bf16(ex, d, inter)
    per = 3 * inter * d
    assert out.size == 2 * per
    for e in range(2):
        g, u, dn = ex[e]
        for i in (0, 5, 31):
            for j in (0, 7, 31):
                assert out[e * per + i * 2 * d + j] == g.bits[i, j]
                assert out[e * per + i * 2 * d + d + j] == u.bits[i, j]
        for n in (0, 9, 31):
            for j in (0, 16, 31):
                assert out[e * per + 2 * inter * d + n * inter + j] == dn.bits[n, j]
    # every element placed exactly once
    assert np.array_equal(np.sort(out), np.sort(np.concatenate([m.bits.ravel() for t in ex for m in t])))
