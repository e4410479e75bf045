"""Pins of the oracle's attention prologue (fused Q/K RMS normalisation +
rotary embedding + key/value pass-through) against properties the
mathematics fixes: the RMS of a normalised head, the direction it keeps, the
per-projection weights, the rotations by 0, 90 and 180 degrees (which fix the
pairing (i, i + Dh/2) and the signs), the length of every rotated pair, the
table row each token's position selects, value heads passed bit for bit, and
an all-zero head."""
import numpy as np

import oracle
import synth

HQ, HKV, DH = 4, 2, 128


def _qkv(seed, T, scale=1.0):
    rng = np.random.default_rng(seed)
    return synth.to_bf16_bits((rng.standard_normal((T, HQ + 2 * HKV, DH)) * scale).astype(np.float32))


def _w(val):
    return synth.to_bf16_bits(np.full(DH, val, np.float32))


def _table(angles):
    """cos/sin rows for the given angle per row (the same angle for every pair)."""
    a = np.asarray(angles, np.float64)[:, None] * np.ones((1, DH // 2))
    return np.concatenate([np.cos(a), np.sin(a)], axis=1).astype(np.float32)


def test_norm_rms_and_direction():
    x_bits = _qkv(1, 3, scale=0.37)
    q, k, _ = oracle.qk_norm_rope_kv(x_bits, HQ, HKV, _w(1.0), _w(1.0), eps=1e-6)
    x = synth.bf16_bits_to_f64(x_bits)
    for t in range(3):
        for h in range(HQ + HKV):
            xh = x[t, h]
            y = q[t, h] if h < HQ else k[t, h - HQ]
            ms = np.mean(xh ** 2)
            # mean(y^2) = mean(x^2) / (mean(x^2) + eps)
            assert abs(np.sqrt(np.mean(y ** 2)) - np.sqrt(ms / (ms + 1e-6))) < 1e-12
            # same direction as x
            assert abs(np.dot(xh, y) / (np.linalg.norm(xh) * np.linalg.norm(y)) - 1.0) < 1e-12


def test_weights_per_projection():
    x_bits = _qkv(2, 2)
    q1, k1, _ = oracle.qk_norm_rope_kv(x_bits, HQ, HKV, _w(1.0), _w(1.0))
    q2, k3, _ = oracle.qk_norm_rope_kv(x_bits, HQ, HKV, _w(2.0), _w(3.0))
    assert np.array_equal(q2, 2.0 * q1) and np.array_equal(k3, 3.0 * k1)
    # an elementwise weight scales its own element only
    w = np.ones(DH, np.float32)
    w[5] = 0.5
    q5, _, _ = oracle.qk_norm_rope_kv(x_bits, HQ, HKV, synth.to_bf16_bits(w), _w(1.0))
    assert np.allclose(q5[..., 5], 0.5 * q1[..., 5], rtol=0, atol=1e-15)
    assert np.array_equal(np.delete(q5, 5, axis=-1), np.delete(q1, 5, axis=-1))


def test_rotation_identity_quarter_half_turn():
    x_bits = _qkv(3, 3)
    base_q, base_k, _ = oracle.qk_norm_rope_kv(x_bits, HQ, HKV, _w(1.0), _w(1.0))
    h = DH // 2
    # rows 0, 1, 2: cos/sin of 0, 90 and 180 degrees (exactly 1/0, 0/1, -1/0)
    cs = np.zeros((3, DH), np.float32)
    cs[0, :h] = 1.0
    cs[1, h:] = 1.0
    cs[2, :h] = -1.0
    for t, pos in enumerate([0, 1, 2]):
        positions = np.full(3, pos, np.int32)
        q, k, _ = oracle.qk_norm_rope_kv(x_bits, HQ, HKV, _w(1.0), _w(1.0), cs, positions, rope=True)
        for out, base in ((q, base_q), (k, base_k)):
            if pos == 0:
                assert np.array_equal(out, base)
            elif pos == 1:  # (a, b) -> (-b, a)
                assert np.array_equal(out[..., :h], -base[..., h:])
                assert np.array_equal(out[..., h:], base[..., :h])
            else:
                assert np.array_equal(out, -base)


def test_rotation_keeps_pair_lengths_and_uses_the_position_row():
    x_bits = _qkv(4, 4)
    base_q, _, _ = oracle.qk_norm_rope_kv(x_bits, HQ, HKV, _w(1.0), _w(1.0))
    angles = np.linspace(0.1, 2.9, 8)
    cs = _table(angles)
    positions = np.array([7, 0, 3, 3], np.int32)
    q, _, _ = oracle.qk_norm_rope_kv(x_bits, HQ, HKV, _w(1.0), _w(1.0), cs, positions, rope=True)
    h = DH // 2
    for t in range(4):
        a0, b0 = base_q[t, :, :h], base_q[t, :, h:]
        a1, b1 = q[t, :, :h], q[t, :, h:]
        assert np.allclose(a1 ** 2 + b1 ** 2, a0 ** 2 + b0 ** 2, rtol=1e-6, atol=1e-12)
        # the angle between (a0, b0) and (a1, b1) is the row's angle (counter-clockwise)
        ang = np.arctan2(a0 * b1 - b0 * a1, a0 * a1 + b0 * b1)
        assert np.allclose(ang, angles[positions[t]], atol=1e-5)


def test_values_pass_and_zero_heads():
    x_bits = _qkv(5, 2)
    _, _, v = oracle.qk_norm_rope_kv(x_bits, HQ, HKV, _w(1.0), _w(1.0))
    assert np.array_equal(v, synth.bf16_bits_to_f64(x_bits)[:, HQ + HKV:])
    z = np.zeros((1, HQ + 2 * HKV, DH), np.uint16)
    q, k, v = oracle.qk_norm_rope_kv(z, HQ, HKV, _w(1.0), _w(1.0), eps=1e-6)
    assert not q.any() and not k.any() and not v.any()
