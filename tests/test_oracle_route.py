"""Pins of the oracle's router: top-k by brute force over every k-subset,
crafted ties, zero inputs, and the gate invariants."""
import itertools
import math

import numpy as np
import pytest

import oracle


def _brute_topk(logits, k):
    """The unique k-subset S such that every selected expert beats every
    unselected one under (larger logit, then lower index); returned in that order."""
    E = len(logits)
    beats = lambda i, j: logits[i] > logits[j] or (logits[i] == logits[j] and i < j)
    found = []
    for S in itertools.combinations(range(E), k):
        rest = [j for j in range(E) if j not in S]
        if all(beats(i, j) for i in S for j in rest):
            found.append(S)
    assert len(found) == 1
    S = list(found[0])
    # order inside S: selection order = sorted by the same relation
    for a in range(k):
        for b in range(a + 1, k):
            if beats(S[b], S[a]):
                S[a], S[b] = S[b], S[a]
    return S


@pytest.mark.parametrize("E,k", [(6, 6), (8, 2), (10, 6), (12, 6), (12, 3)])
def test_topk_brute_force_small(E, k):
    rng = np.random.default_rng(E * 10 + k)
    for trial in range(20):
        # coarse values so that exact ties happen often
        logits = rng.integers(-3, 4, size=(1, E)).astype(np.float64) * 0.5
        ids, gates, gap = oracle.topk(logits, k)
        assert list(ids[0]) == _brute_topk(logits[0], k)
        p = np.exp(logits[0] - logits[0].max())
        p /= p.sum()
        np.testing.assert_allclose(gates[0], p[ids[0]] / p[ids[0]].sum(), rtol=1e-14)
        assert abs(gates[0].sum() - 1.0) <= 1e-12


def test_topk_random_e32_matches_stable_sort():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((50, 32))
    ids, gates, gap = oracle.topk(logits, 6)
    for t in range(50):
        order = sorted(range(32), key=lambda e: (-logits[t, e], e))
        assert list(ids[t]) == order[:6]
        p = np.exp(logits[t] - logits[t].max())
        p /= p.sum()
        assert gap[t] == pytest.approx(p[order[5]] - p[order[6]], abs=1e-15)


def test_all_equal_logits_pick_lowest_indices():
    ids, gates, gap = oracle.topk(np.full((2, 32), 0.75), 6)
    assert ids.tolist() == [[0, 1, 2, 3, 4, 5]] * 2
    np.testing.assert_allclose(gates, 1 / 6, rtol=0, atol=1e-15)
    assert gap.tolist() == [0.0, 0.0]


def test_signed_zero_logits_tie():
    logits = np.array([[-0.0, 0.0, -0.0, 0.0, -1.0, 0.0, -0.0, -2.0]])
    ids, _, _ = oracle.topk(logits, 6)
    assert ids[0].tolist() == [0, 1, 2, 3, 5, 6]


def test_zero_input_gives_first_experts_equal_gates():
    x = np.zeros((3, 64), np.uint16)
    rng = np.random.default_rng(1)
    import synth
    wr = synth.to_bf16_bits(rng.standard_normal((32, 64)) * 0.02)
    logits = oracle.router_logits(x, wr)
    assert not logits.any()
    ids, gates, _ = oracle.topk(logits, 6)
    assert ids.tolist() == [[0, 1, 2, 3, 4, 5]] * 3
    np.testing.assert_allclose(gates, 1 / 6, atol=1e-15)


def test_router_logits_exact_small_integers():
    # bf16 integers: the fp64 dot product is exact
    import synth
    x = synth.to_bf16_bits(np.array([[1, 2, 3, 4, 0, -1, 5, 7]], np.float32))
    wr = synth.to_bf16_bits(np.array([[1, 0, 0, 0, 0, 0, 0, 0], [1, 1, 1, 1, 1, 1, 1, 1],
                                      [0, 0, 0, 0, 0, 0, 0, -2]], np.float32))
    assert oracle.router_logits(x, wr).tolist() == [[1.0, 21.0, -14.0]]


def test_k_equals_e_gap_infinite_and_gates_full_softmax():
    logits = np.array([[0.1, -0.3, 2.0, 0.0]])
    ids, gates, gap = oracle.topk(logits, 4)
    assert ids[0].tolist() == [2, 0, 3, 1]
    p = np.exp(logits[0] - 2.0)
    p /= p.sum()
    np.testing.assert_allclose(gates[0], p[[2, 0, 3, 1]], rtol=1e-14)
    assert math.isinf(gap[0])
