"""Pins of the oracle's element codecs (E2M1, E4M3, bf16 rounding).

Decoders are pinned to every code of the format tables; encoders are pinned to
an exhaustive nearest-value search (a different algorithm from the oracle's
binade arithmetic) and to hand-worked tie cases.
"""
import math

import numpy as np
import pytest

import oracle
from conftest import golden


def test_e2m1_every_code_matches_table():
    rows = golden("e2m1_codes.txt")
    assert len(rows) == 16
    for code_s, val_s in rows:
        code, val = int(code_s, 16), float(val_s)
        got = oracle.e2m1_decode(code)
        assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), (code, got, val)


def test_e4m3_edge_codes():
    for code_s, val_s in golden("e4m3_edges.txt"):
        code = int(code_s, 16)
        got = oracle.e4m3_decode(code)
        if val_s == "nan":
            assert math.isnan(got)
        else:
            val = float(val_s)
            assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), (code, got)


def test_e4m3_all_finite_codes_monotone_and_distinct():
    vals = [oracle.e4m3_decode(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(vals, vals[1:]))
    assert vals[-1] == 448.0


def test_nvfp4_products():
    for q_s, sb_s, st_s, val_s in golden("nvfp4_products.txt"):
        got = oracle.e2m1_decode(int(q_s, 16)) * oracle.e4m3_decode(int(sb_s, 16)) * float(st_s)
        assert got == float(val_s)


def _nearest_even(a, table):
    """Exhaustive search: index of the nearest table value to a; on a tie the
    index with an even code (mantissa bit 0)."""
    best, best_d = None, None
    for i, v in enumerate(table):
        d = abs(a - v)
        if best is None or d < best_d or (d == best_d and i % 2 == 0 and best % 2 == 1):
            best, best_d = i, d
    return best


E2M1_MAG = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_encode_brute_force():
    rng = np.random.default_rng(0)
    vals = np.concatenate([np.linspace(-7, 7, 2801), rng.uniform(-8, 8, 5000)]).astype(np.float32)
    for v in vals:
        code = oracle.e2m1_encode(float(v))
        a = min(abs(float(v)), 6.0)
        want = _nearest_even(a, E2M1_MAG)
        assert code & 7 == want, (float(v), code)
        assert (code >> 3) == (1 if np.signbit(v) else 0)


@pytest.mark.parametrize("v,code", [(0.25, 0x0), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4),
                                    (3.5, 0x6), (5.0, 0x6), (5.5, 0x7), (7.0, 0x7), (1e9, 0x7),
                                    (-0.25, 0x8), (-0.0, 0x8), (0.0, 0x0), (-5.0, 0xE),
                                    (0.2499, 0x0), (0.2501, 0x1)])
def test_e2m1_ties_and_saturation(v, code):
    assert oracle.e2m1_encode(v) == code


def test_e4m3_encode_brute_force():
    table = [oracle.e4m3_decode(c) for c in range(0x7F)]
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        np.array([0.0, 2.0 ** -10, 3 * 2.0 ** -11, 7.5 * 2.0 ** -9, 447.9, 448.0, 460.0, 1e6]),
        np.exp(rng.uniform(np.log(1e-4), np.log(500), 20000)),
        (np.arange(0, 300) * 2.0 ** -12),
    ]).astype(np.float32)
    for v in vals:
        code = oracle.e4m3_encode(float(v))
        want = _nearest_even(min(float(v), 448.0), table)
        assert code == want, (float(v), hex(code), hex(want))


@pytest.mark.parametrize("v,code", [(2.0 ** -10, 0x00), (3 * 2.0 ** -10, 0x02), (7.5 * 2.0 ** -9, 0x08),
                                    (1.0625, 0x38), (1.1875, 0x3A), (464.0, 0x7E), (1e30, 0x7E)])
def test_e4m3_ties(v, code):
    assert oracle.e4m3_encode(v) == code


@pytest.mark.parametrize("v,bits", [(1.0, 0x3F80), (-2.0, 0xC000), (1.0 + 2 ** -8, 0x3F80),
                                    (1.0 + 3 * 2 ** -8, 0x3F82), (1.0 + 2 ** -8 + 2 ** -30, 0x3F81),
                                    (0.0, 0x0000), (-0.0, 0x8000), (3.0e38, 0x7F62),
                                    (3.4e38, 0x7F80), (2.0 ** -133, 0x0001), (2.0 ** -134, 0x0000)])
def test_bf16_round_nearest_even(v, bits):
    assert oracle.bf16_from_double(v) == bits


def test_bf16_matches_fp32_cast_on_fp32_values():
    # for values exactly representable in fp32, RNE to bf16 equals torch's fp32->bf16 cast
    import torch
    rng = np.random.default_rng(2)
    a = rng.standard_normal(2000).astype(np.float32) * np.float32(3.0)
    want = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_round_array(a.astype(np.float64))
    assert np.array_equal(got, want)
