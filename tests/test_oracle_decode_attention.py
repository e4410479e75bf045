"""Pins of the oracle's decode attention: against PyTorch's scaled dot-product
attention in float64 on the same cache slice (a library routine for the
special case of one query per head), a single key (the output is that key's
value), identical keys (the mean of the values), the grouped-query mapping
(query head h reads key/value head h / (Hq / Hkv) and no other), an empty
range (zeros), and the row range each token's start selects."""
import numpy as np
import torch

import oracle
import synth

HQ, HKV, DH = 8, 2, 16


def _bits(seed, shape, scale=1.0):
    rng = np.random.default_rng(seed)
    return synth.to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def test_matches_library_sdpa_in_float64():
    T, rows = 3, 50
    q, k, v = _bits(1, (T, HQ, DH)), _bits(2, (rows, HKV, DH)), _bits(3, (rows, HKV, DH))
    start = np.array([0, 10, 33], np.int64)
    length = np.array([50, 17, 5], np.int32)
    got = oracle.decode_attention(q, k, v, start, length)
    qf, kf, vf = (torch.from_numpy(synth.bf16_bits_to_f64(a)) for a in (q, k, v))
    for t in range(T):
        ks = kf[start[t]:start[t] + length[t]].permute(1, 0, 2)  # [Hkv][L][Dh]
        vs = vf[start[t]:start[t] + length[t]].permute(1, 0, 2)
        ks = ks.repeat_interleave(HQ // HKV, dim=0)
        vs = vs.repeat_interleave(HQ // HKV, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qf[t][:, None, :], ks, vs)[:, 0, :].numpy()
        assert np.allclose(got[t], ref, rtol=1e-12, atol=1e-13)


def test_single_key_and_identical_keys():
    q, k, v = _bits(4, (1, HQ, DH)), _bits(5, (6, HKV, DH)), _bits(6, (6, HKV, DH))
    out = oracle.decode_attention(q, k, v, np.array([4], np.int64), np.array([1], np.int32))
    vv = synth.bf16_bits_to_f64(v)
    for h in range(HQ):
        assert np.array_equal(out[0, h], vv[4, h // (HQ // HKV)])
    k_same = np.repeat(k[:1], 6, axis=0)
    out = oracle.decode_attention(q, k_same, v, np.array([0], np.int64), np.array([6], np.int32))
    for h in range(HQ):
        assert np.allclose(out[0, h], vv[:, h // (HQ // HKV)].mean(axis=0), rtol=0, atol=1e-15)


def test_grouped_query_mapping_and_empty_range():
    q, k, v = _bits(7, (2, HQ, DH)), _bits(8, (9, HKV, DH)), _bits(9, (9, HKV, DH))
    start, length = np.array([0, 3], np.int64), np.array([9, 0], np.int32)
    base = oracle.decode_attention(q, k, v, start, length)
    k2, v2 = k.copy(), v.copy()
    k2[:, 0] = _bits(10, (9, DH))
    v2[:, 0] = _bits(11, (9, DH))
    pert = oracle.decode_attention(q, k2, v2, start, length)
    g = HQ // HKV
    assert np.array_equal(pert[:, g:], base[:, g:])            # heads of kv head 1: unchanged
    assert not np.allclose(pert[0, :g], base[0, :g])          # heads of kv head 0: changed
    assert not base[1].any()                                  # empty range: zeros


def test_shift_of_every_key_leaves_the_output_unchanged():
    # adding one vector c to every key adds q . c to all of a head's scores:
    # the softmax, and so the output, stay the same. Keys on a coarse grid so
    # that k + c is exact in bf16.
    rng = np.random.default_rng(12)
    L = 40
    q = _bits(13, (2, HQ, DH))
    k = synth.to_bf16_bits(rng.integers(-8, 8, (L, HKV, DH)).astype(np.float32) / 4)
    c = rng.integers(-4, 4, (1, HKV, DH)).astype(np.float32) / 4
    k2 = synth.to_bf16_bits(synth.bf16_bits_to_f64(k).astype(np.float32) + c)
    v = _bits(14, (L, HKV, DH))
    start, length = np.array([0, 5], np.int64), np.array([40, 30], np.int32)
    a = oracle.decode_attention(q, k, v, start, length)
    b = oracle.decode_attention(q, k2, v, start, length)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-13)


def test_linear_in_the_values_and_blind_to_row_order():
    q, k, v = _bits(15, (1, HQ, DH)), _bits(16, (25, HKV, DH)), _bits(17, (25, HKV, DH))
    start, length = np.array([0], np.int64), np.array([25], np.int32)
    base = oracle.decode_attention(q, k, v, start, length)
    v4 = synth.to_bf16_bits(synth.bf16_bits_to_f64(v).astype(np.float32) * 4)  # exact
    assert np.allclose(oracle.decode_attention(q, k, v4, start, length), 4 * base, rtol=1e-13, atol=0)
    perm = np.random.default_rng(18).permutation(25)
    got = oracle.decode_attention(q, k[perm], v[perm], start, length)
    assert np.allclose(got, base, rtol=1e-12, atol=1e-14)


def test_scale_argument_sharpens_toward_the_best_key():
    # a large score scale turns the softmax into an argmax: each head's output
    # becomes the value row of its highest-scoring key
    q, k, v = _bits(19, (1, HQ, DH)), _bits(20, (12, HKV, DH)), _bits(21, (12, HKV, DH))
    start, length = np.array([0], np.int64), np.array([12], np.int32)
    out = oracle.decode_attention(q, k, v, start, length, scale=1e4)
    qf, kf, vf = (synth.bf16_bits_to_f64(a) for a in (q, k, v))
    g = HQ // HKV
    for h in range(HQ):
        s = kf[:, h // g] @ qf[0, h]
        best = int(np.argmax(s))
        assert np.sort(s)[-1] - np.sort(s)[-2] > 1e-2  # a clear winner at this seed
        assert np.allclose(out[0, h], vf[best, h // g], rtol=0, atol=1e-12)
