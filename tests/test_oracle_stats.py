"""Pins for the oracle's routing statistics: per-expert routing counts and the
smallest covering expert set (CMF code specialist page, How it was made:
Calibrate and Defrag steps)."""
import itertools

import numpy as np
import pytest

import oracle


def test_counts_equal_bincount_and_skip_invalid():
    rng = np.random.default_rng(0)
    E = 37
    idx = rng.integers(-3, E + 3, size=(211, 8)).astype(np.int32)
    got = oracle.expert_counts(idx, E)
    valid = idx[(idx >= 0) & (idx < E)]
    np.testing.assert_array_equal(got, np.bincount(valid, minlength=E).astype(np.uint64))


def test_counts_accumulate_across_calls():
    rng = np.random.default_rng(1)
    a = rng.integers(0, 16, size=(50, 4)).astype(np.int32)
    b = rng.integers(0, 16, size=(70, 4)).astype(np.int32)
    c = oracle.expert_counts(a, 16)
    oracle.expert_counts(b, 16, counts=c)
    np.testing.assert_array_equal(c, oracle.expert_counts(np.concatenate([a, b]), 16))


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("cover", [0.5, 0.8, 0.95, 1.0])
def test_cover_set_is_a_smallest_cover_brute_force(seed, cover):
    """No smaller subset reaches cover * total, and among sets of the chosen size the
    kept one carries the most mass (so it is the greedy prefix up to ties)."""
    rng = np.random.default_rng(seed)
    E = 9
    counts = rng.integers(0, 12, size=E).astype(np.uint64)
    counts[rng.integers(E)] = 0
    keep, new_index, n = oracle.cover_set(counts, cover)
    total = float(counts.sum())
    target = cover * total
    kept = np.nonzero(keep)[0]
    assert kept.size == n and float(counts[kept].sum()) >= target
    best = {}
    for m in range(E + 1):
        for sub in itertools.combinations(range(E), m):
            s = float(counts[list(sub)].sum())
            if s >= target:
                best.setdefault(m, s)
                best[m] = max(best[m], s)
    m_min = min(best)
    assert n == m_min
    assert float(counts[kept].sum()) == best[m_min]


def test_cover_ties_keep_the_lower_index_and_renumber_densely():
    counts = np.array([4, 7, 4, 0, 7, 4], np.uint64)  # total 26; 0.6 * 26 = 15.6
    keep, new_index, n = oracle.cover_set(counts, 0.6)
    assert n == 3 and keep.tolist() == [1, 1, 0, 0, 1, 0]
    assert new_index.tolist() == [0, 1, -1, -1, 2, -1]


def test_full_cover_keeps_exactly_the_used_experts():
    counts = np.array([0, 3, 0, 1, 9, 0, 2], np.uint64)
    keep, new_index, n = oracle.cover_set(counts, 1.0)
    assert keep.tolist() == [int(c > 0) for c in counts] and n == 4
    assert sorted(new_index[new_index >= 0].tolist()) == list(range(4))


def test_cover_rejects_out_of_range_share():
    with pytest.raises(ValueError):
        oracle.cover_set(np.ones(4, np.uint64), 0.0)
    with pytest.raises(ValueError):
        oracle.cover_set(np.ones(4, np.uint64), 1.5)
