"""Pins of the oracle's expert-parallel dispatch plan: a small case worked out
by hand, and on random routings the properties that fix the plan -- every
valid pair sent exactly once, to the rank that holds its expert, with the
local id that names that expert there, shared slots kept on the home rank,
destination ranks in ascending order and pair order kept within a rank,
counts that add up, and ids outside [0, E) dropped."""
import numpy as np

import oracle


def test_hand_worked_case():
    # E = 4 experts on R = 2 ranks (rank 0: experts 0, 1; rank 1: 2, 3), top-2
    # plus one shared expert, planned on rank 1.
    ids = np.array([[3, 0], [1, 2]], np.int32)
    gates = np.array([[0.75, 0.25], [0.5, 0.5]], np.float32)
    p = oracle.ep_plan(ids, gates, S=1, E=4, R=2, rank=1)
    # pairs: 0 (t0, e3 -> r1), 1 (t0, e0 -> r0), 2 (t0 shared -> r1),
    #        3 (t1, e1 -> r0), 4 (t1, e2 -> r1), 5 (t1 shared -> r1)
    assert p["counts"].tolist() == [2, 4]
    assert p["pair_pos"].ravel().tolist() == [2, 0, 3, 1, 4, 5]
    assert p["send_ids"].tolist() == [0, 1, 1, 2, 0, 2]      # local ids; the shared expert is E/R = 2
    assert p["send_token"].tolist() == [0, 1, 0, 0, 1, 1]
    assert p["send_gates"].tolist() == [0.25, 0.5, 0.75, 1.0, 0.5, 1.0]
    assert p["dropped"] == 0


def test_random_plans_properties():
    rng = np.random.default_rng(0)
    for R, E, k, S, T in [(1, 8, 2, 1, 5), (2, 256, 6, 1, 33), (4, 256, 6, 1, 64), (8, 256, 6, 0, 100),
                          (8, 64, 8, 1, 7)]:
        ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        gates = rng.random((T, k)).astype(np.float32)
        rank = int(rng.integers(R))
        p = oracle.ep_plan(ids, gates, S=S, E=E, R=R, rank=rank)
        el = E // R
        slots = k + S
        assert p["counts"].sum() == T * slots == len(p["send_ids"])
        pos = p["pair_pos"].ravel()
        assert sorted(pos.tolist()) == list(range(T * slots))            # a permutation
        bounds = np.concatenate([[0], np.cumsum(p["counts"])])
        for i in range(T * slots):
            t, j = divmod(i, slots)
            q = pos[i]
            r = int(np.searchsorted(bounds, q, side="right") - 1)        # rank of the send slot
            assert p["send_token"][q] == t
            if j < k:
                assert r * el + p["send_ids"][q] == ids[t, j]             # the expert, on its rank
                assert p["send_gates"][q] == gates[t, j]
            else:
                assert r == rank and p["send_ids"][q] == el + (j - k) and p["send_gates"][q] == 1.0
        # pair order kept within each destination rank
        for r in range(R):
            src = [i for i in range(T * slots) if bounds[r] <= pos[i] < bounds[r + 1]]
            assert [pos[i] for i in src] == list(range(bounds[r], bounds[r + 1]))


def test_out_of_range_ids_are_dropped():
    ids = np.array([[0, 9], [-1, 5]], np.int32)
    gates = np.ones((2, 2), np.float32)
    p = oracle.ep_plan(ids, gates, S=0, E=8, R=2, rank=0)
    assert p["dropped"] == 2
    assert p["pair_pos"].ravel().tolist() == [0, -1, -1, 1]
    assert p["counts"].tolist() == [1, 1] and p["send_ids"].tolist() == [0, 1]
