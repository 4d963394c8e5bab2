"""Pins of the oracle's baseline selectors (recency only, random fraction of the older chunks).

The random selector is checked against a sequential restatement of the published
SplitMix64 generator (the counter form the oracle uses must give the same outputs as
stepping the generator), against numpy's lexicographic sort for the choice of the
smallest draws, against the rounding rule for the count, and statistically for
uniformity over many seeds.
"""
import numpy as np

import oracle

GAMMA = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1


def splitmix64_stream(seed, n):
    """First n outputs of SplitMix64 started at `seed`, stepped one output at a time."""
    state, out = seed & M64, []
    for _ in range(n):
        state = (state + GAMMA) & M64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
        out.append(z ^ (z >> 31))
    return out


def test_recency_only_keeps_no_older_chunk(oracle_mod):
    ws = np.array([0, 64, 8000 * 64, 123 * 64], np.int32)
    kept, rc, cnt = oracle_mod.select_baseline(oracle.RECENT, ws, seed=3)
    assert rc == 0 and cnt.tolist() == [0, 0, 0, 0] and all(k.size == 0 for k in kept)


def test_random_selection_is_the_smallest_sequential_splitmix_draws(oracle_mod):
    """Sequence 0's draws are outputs 0..n-1 of the stream; the kept chunks are the m with the
    smallest top-24-bit draws, ties to the lower index."""
    for seed, n_old in ((0, 300), (12345, 77), (2 ** 63 + 7, 1000)):
        draws = np.array([x >> 40 for x in splitmix64_stream(seed, n_old)], np.int64)
        m = (n_old + 5) // 10
        ref = np.sort(np.lexsort((np.arange(n_old), draws))[:m])
        kept, rc, cnt = oracle_mod.select_baseline(oracle.RANDOM, np.array([n_old * 64], np.int32), seed=seed)
        assert rc == 0 and cnt[0] == m
        np.testing.assert_array_equal(kept[0], ref)


def test_random_count_rounds_half_up_and_respects_the_fraction(oracle_mod):
    # n_old = 25 at 1/10 is 2.5 -> 3; 24 -> 2.4 -> 2; 3/8 of 12 = 4.5 -> 5; 0 -> 0; all of 7 -> 7
    cases = [(25, 1, 10, 3), (24, 1, 10, 2), (12, 3, 8, 5), (0, 1, 10, 0), (7, 1, 1, 7), (7, 0, 1, 0)]
    for n_old, num, den, m in cases:
        kept, rc, cnt = oracle_mod.select_baseline(oracle.RANDOM, np.array([n_old * 64], np.int32), seed=9,
                                                   keep_num=num, keep_den=den)
        assert cnt[0] == m, (n_old, num, den)
        assert np.all(np.diff(kept[0]) > 0) and (kept[0].size == 0 or (kept[0].min() >= 0 and kept[0].max() < n_old))


def test_random_selection_is_uniform_over_seeds(oracle_mod):
    """Over 3000 seeds every one of 40 chunks is kept with frequency close to 4/40."""
    n_old, seeds = 40, 3000
    freq = np.zeros(n_old)
    for seed in range(seeds):
        kept, _, cnt = oracle_mod.select_baseline(oracle.RANDOM, np.array([n_old * 64], np.int32), seed=seed)
        assert cnt[0] == 4
        freq[kept[0]] += 1
    expected = seeds * 4 / n_old
    chi2 = float(((freq - expected) ** 2 / expected).sum())
    assert chi2 < 90.0          # 39 degrees of freedom: the 1e-5 upper quantile is about 89


def test_random_sequences_draw_from_their_own_counters(oracle_mod):
    ws = np.array([500 * 64, 500 * 64], np.int32)
    kept, _, cnt = oracle_mod.select_baseline(oracle.RANDOM, ws, seed=1)
    assert cnt.tolist() == [50, 50] and not np.array_equal(kept[0], kept[1])
    alone, _, _ = oracle_mod.select_baseline(oracle.RANDOM, ws[:1], seed=1)
    np.testing.assert_array_equal(alone[0], kept[0])
