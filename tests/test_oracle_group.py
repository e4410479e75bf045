"""Pins of the oracle's grouping by expert (the expert histogram and token
permutation of the layer contract): every (token, slot) selection appears
exactly once, under its expert; experts ascend; each expert's tokens ascend;
offsets are the running counts; the shared experts serve every token last;
brute-force counts against numpy's histogram; out-of-range ids are refused."""
import itertools

import numpy as np
import pytest

import oracle


def _random_ids(rng, T, E, k):
    return np.array([rng.choice(E, size=k, replace=False) for _ in range(T)], dtype=np.int32).reshape(T, k)


def _check_invariants(ids, E, S, res):
    act, off, pair, nr = res
    T, k = ids.shape
    n = len(act)
    assert n == nr + S
    assert np.all(np.diff(act[:nr]) > 0) and np.all((act[:nr] >= 0) & (act[:nr] < E))
    assert act[nr:].tolist() == list(range(E, E + S))
    assert off[0] == 0 and off[-1] == T * (k + S) and np.all(np.diff(off) > 0)
    hist = np.bincount(ids.ravel(), minlength=E)
    assert sorted(act[:nr].tolist()) == np.nonzero(hist)[0].tolist()
    seen = set()
    for a in range(n):
        ps = pair[off[a]:off[a + 1]]
        toks = ps >> 8
        assert np.all(np.diff(toks) > 0)  # one selection per token, ascending
        for p in ps.tolist():
            t, j = p >> 8, p & 0xFF
            if a < nr:
                assert off[a + 1] - off[a] == hist[act[a]]
                assert ids[t, j] == act[a]
            else:
                assert j == k + (a - nr)
            assert (t, j) not in seen
            seen.add((t, j))
    assert len(seen) == T * (k + S)


@pytest.mark.parametrize("T,E,k,S", [(1, 256, 6, 1), (4, 32, 6, 1), (8, 256, 6, 1), (13, 40, 6, 0),
                                     (64, 256, 6, 1), (128, 256, 6, 1), (7, 8, 8, 1), (3, 1, 1, 0)])
def test_grouping_invariants_random(T, E, k, S):
    rng = np.random.default_rng(T * 1000 + E + k)
    for _ in range(3):
        ids = _random_ids(rng, T, E, k)
        _check_invariants(ids, E, S, oracle.group(ids, E, S))


def test_grouping_extremes():
    # every token on the same 6 experts: 6 active experts with 128 tokens each
    ids = np.tile(np.array([200, 3, 77, 150, 9, 255], np.int32), (128, 1))
    act, off, pair, nr = oracle.group(ids, 256, 1)
    assert nr == 6 and act.tolist() == [3, 9, 77, 150, 200, 255, 256]
    assert np.diff(off).tolist() == [128] * 7
    slot_of = {e: j for j, e in enumerate([200, 3, 77, 150, 9, 255])}
    for a, e in enumerate(act[:6].tolist()):
        assert pair[off[a]:off[a + 1]].tolist() == [(t << 8) | slot_of[e] for t in range(128)]
    # every selection on a distinct expert: 192 active experts of one pair each
    ids = np.arange(32 * 6, dtype=np.int32)[::-1].reshape(32, 6).copy()
    act, off, pair, nr = oracle.group(ids, 256, 1)
    assert nr == 192 and act[:192].tolist() == list(range(192))
    for a in range(192):
        t, j = divmod(191 - a, 6)
        assert pair[off[a]:off[a + 1]].tolist() == [(t << 8) | j]


def test_grouping_brute_force_tiny():
    # all selections of T=2 tokens, k=2 of E=4: pairs sorted by (expert, token)
    for a0, a1 in itertools.permutations(range(4), 2):
        for b0, b1 in itertools.permutations(range(4), 2):
            ids = np.array([[a0, a1], [b0, b1]], np.int32)
            act, off, pair, nr = oracle.group(ids, 4, 0)
            sel = sorted((int(ids[t, j]), t, j) for t in range(2) for j in range(2))
            assert pair.tolist() == [(t << 8) | j for _, t, j in sel]
            assert act.tolist() == sorted(set(e for e, _, _ in sel))


@pytest.mark.parametrize("bad", [-1, 256, 1 << 20])
def test_grouping_refuses_out_of_range_ids(bad):
    ids = np.array([[1, 2, bad, 4, 5, 6]], np.int32)
    assert oracle.group(ids, 256, 1) is None
