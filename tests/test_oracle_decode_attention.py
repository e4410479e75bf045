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
