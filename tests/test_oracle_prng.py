"""Pins for the oracle's counter-based generator and its without-replacement draw."""
import os
from collections import Counter

import numpy as np

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "splitmix64.txt")


def _golden():
    rows, cur = {}, None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("seed"):
            cur = int(line.split()[1])
            rows[cur] = []
        else:
            rows[cur].append(int(line, 0))
    return rows


def test_splitmix64_published_vectors():
    for seed, expect in _golden().items():
        g = O.SplitMix64(seed)
        assert [g.next() for _ in expect] == expect


def test_streams_differ_and_are_reproducible():
    a = O.SplitMix64(O.stream_state(7, 3, 1))
    b = O.SplitMix64(O.stream_state(7, 3, 1))
    c = O.SplitMix64(O.stream_state(7, 3, 2))
    xa = [a.next() for _ in range(8)]
    assert xa == [b.next() for _ in range(8)]
    assert xa != [c.next() for _ in range(8)]


def test_draw_is_a_partial_fisher_yates():
    # drawing all n items is a permutation; the prefix of a longer draw equals a
    # shorter draw from the same stream state
    for n in (1, 2, 5, 17, 64):
        full = O.draw_without_replacement(O.SplitMix64(99), n, n)
        assert sorted(full) == list(range(n))
        for m in range(n + 1):
            assert O.draw_without_replacement(O.SplitMix64(99), n, m) == full[:m]


def test_draw_matches_explicit_array_shuffle():
    # the sparse slot map must equal a dense array shuffled in place
    rng_a, rng_b = O.SplitMix64(5), O.SplitMix64(5)
    n, m = 50, 20
    arr = list(range(n))
    dense = []
    for i in range(m):
        j = i + rng_b.next() % (n - i)
        arr[i], arr[j] = arr[j], arr[i]
        dense.append(arr[i])
    assert O.draw_without_replacement(rng_a, n, m) == dense


def test_draw_is_uniform():
    # first item of a draw over 8 items: chi-square against uniform
    n, trials = 8, 16000
    g = O.SplitMix64(2024)
    cnt = Counter(O.draw_without_replacement(g, n, 3)[0] for _ in range(trials))
    exp = trials / n
    chi2 = sum((cnt[i] - exp) ** 2 / exp for i in range(n))
    assert chi2 < 24.3  # p ~ 0.001 for 7 dof
    # every pair equally likely to be drawn together
    pairs = Counter()
    for _ in range(6000):
        a, b = O.draw_without_replacement(g, 5, 2)
        pairs[frozenset((a, b))] += 1
    vals = np.array(list(pairs.values()))
    assert len(pairs) == 10 and vals.min() > 0.8 * vals.mean()
