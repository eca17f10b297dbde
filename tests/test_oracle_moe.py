"""Pins of the MoE expand permutation oracle (a stable counting sort of the (token, choice) entries
by expert), against what fixes it independently of its code:

* two examples worked out by hand (the derivation is in the comments);
* a library stable sort (numpy's mergesort-based argsort) of the same keys gives the same order;
* invariants on random routings: the expanded experts are sorted, every placed position is hit
  exactly once, the inverse map points back at the entry, equal experts keep their token order,
  the offsets are the exclusive prefix sums of the per-expert counts, and dropped entries (expert
  outside [0, G)) leave -1 in the tail.
"""
import numpy as np
import pytest

import oracle


def test_hand_worked_example():
    # entries in token-major order: (t0,k0)=2 (t0,k1)=0 (t1,k0)=1 (t1,k1)=2 (t2,k0)=0 (t2,k1)=1
    # expert 0 gets entries 1, 4 (tokens 0, 2) at positions 0, 1; expert 1 entries 2, 5 (tokens 1, 2)
    # at 2, 3; expert 2 entries 0, 3 (tokens 0, 1) at 4, 5
    src, mi, dst, off = oracle.moe_permute(np.array([[2, 0], [1, 2], [0, 1]]), 3)
    assert src.tolist() == [0, 2, 1, 2, 0, 1]
    assert mi.tolist() == [0, 0, 1, 1, 2, 2]
    assert dst.tolist() == [[4, 0], [2, 5], [1, 3]]
    assert off.tolist() == [0, 2, 4, 6]


def test_hand_worked_example_with_dropped_entries():
    # G = 2: entries -1, 1, 1, 5; only the two 1s are placed (tokens 0 and 1), the rest dropped
    src, mi, dst, off = oracle.moe_permute(np.array([[-1, 1], [1, 5]]), 2)
    assert src.tolist() == [0, 1, -1, -1]
    assert mi.tolist() == [1, 1, -1, -1]
    assert dst.tolist() == [[-1, 0], [1, -1]]
    assert off.tolist() == [0, 0, 2]


def random_ids(T, top_k, G, seed, invalid=0.0):
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, G, (T, top_k)).astype(np.int32)
    if invalid > 0:
        bad = rng.random((T, top_k)) < invalid
        ids[bad] = rng.choice(np.array([-1, -7, G, G + 3], np.int32), int(bad.sum()))
    return ids


@pytest.mark.parametrize("T,top_k,G,invalid", [(1, 1, 1, 0.0), (7, 3, 5, 0.2), (500, 8, 64, 0.05),
                                               (300, 2, 4096, 0.0), (64, 4, 3, 1.0)])
def test_matches_a_library_stable_sort(T, top_k, G, invalid):
    ids = random_ids(T, top_k, G, seed=T + G, invalid=invalid)
    src, mi, dst, off = oracle.moe_permute(ids, G)
    flat = ids.ravel()
    valid = (flat >= 0) & (flat < G)
    key = np.where(valid, flat, G)                      # dropped entries sort after every expert
    order = np.argsort(key, kind="stable")
    placed = int(valid.sum())
    assert np.array_equal(src[:placed], (order[:placed] // top_k).astype(np.int32))
    assert np.array_equal(mi[:placed], flat[order[:placed]])
    assert np.all(src[placed:] == -1) and np.all(mi[placed:] == -1)
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(flat[valid], minlength=G))]))


@pytest.mark.parametrize("seed", range(4))
def test_invariants(seed):
    rng = np.random.default_rng(seed)
    T, top_k, G = int(rng.integers(1, 400)), int(rng.integers(1, 9)), int(rng.integers(1, 300))
    ids = random_ids(T, top_k, G, seed=seed, invalid=0.1)
    src, mi, dst, off = oracle.moe_permute(ids, G)
    n = T * top_k
    placed = int(off[G])
    assert np.all(np.diff(mi[:placed]) >= 0)                       # experts sorted
    d = dst.ravel()
    ok = d >= 0
    assert np.array_equal(np.sort(d[ok]), np.arange(placed))       # a permutation of [0, placed)
    t_of = np.repeat(np.arange(T), top_k)
    assert np.array_equal(src[d[ok]], t_of[ok])                    # inverse map points back
    assert np.array_equal(mi[d[ok]], ids.ravel()[ok])
    for g in range(G):                                             # stable: token order kept per expert
        run = src[off[g]:off[g + 1]]
        assert np.all(np.diff(run) >= 0)
        assert off[g + 1] - off[g] == int(np.count_nonzero(ids == g))
    assert np.all(d[~ok] == -1) and np.all(src[placed:n] == -1)
