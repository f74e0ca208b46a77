"""Host-side accounting of bench.py: the bytes an early-exit call streams.

The library takes the row pairs in waves, the last adding the bonus row, and each wave reads
only the sequences that accepted every draft before it. When one row pair of the whole batch
is at least 64 MB the waves are [0, 1), [1, 3), [3, 7), [7, 15), ...; smaller batches take
[0, 2), [2, 10), [10, 42), ...; both cut at K. The schedules below are written out by hand and
walked sequence by sequence, independently of the helper's own loop.
"""

import numpy as np

import bench

SMALL = {0: [(0, 0)], 1: [(0, 1)], 2: [(0, 2)], 7: [(0, 2), (2, 7)],
         15: [(0, 2), (2, 10), (10, 15)]}
LARGE = {0: [(0, 0)], 1: [(0, 1)], 2: [(0, 1), (1, 2)], 7: [(0, 1), (1, 3), (3, 7)],
         15: [(0, 1), (1, 3), (3, 7), (7, 15)]}
MB = 1 << 20


def _walk(n_accepted, waves, sample):
    rows = 0
    for j in n_accepted:
        for w, (lo, hi) in enumerate(waves):
            if j < lo:  # stopped in an earlier wave: nothing more is read
                break
            rows += (hi - lo) * (2 if sample else 1)
            if w == len(waves) - 1:
                rows += 1  # the bonus row
    return rows


def test_wave_schedules_by_batch_size():
    for K, waves in SMALL.items():
        assert bench.early_exit_waves(64, K, 129280, 2, True) == waves     # 33 MB per pair
    for K, waves in LARGE.items():
        assert bench.early_exit_waves(256, K, 262144, 2, True) == waves    # 268 MB per pair
    # the threshold, on the bytes of one pair of the batch (P and Q rows when sampling)
    V = 64 * MB // (2 * 2)
    assert bench.early_exit_waves(1, 7, V, 2, True) == LARGE[7]
    assert bench.early_exit_waves(1, 7, V - 1, 2, True) == SMALL[7]
    assert bench.early_exit_waves(1, 7, V, 2, False) == SMALL[7]
    assert bench.early_exit_waves(1, 7, 2 * V, 2, False) == LARGE[7]


def test_early_exit_bytes_follow_the_wave_schedule():
    rng = np.random.default_rng(0)
    V, es = 1000, 2
    for K in SMALL:
        n = rng.integers(0, K + 1, size=200)
        for sample in (False, True):
            assert bench.early_exit_bytes(n, K, V, es, sample) == \
                _walk(n, SMALL[K], sample) * V * es
    n = rng.integers(0, 16, size=300)  # 300 x 2 x 256 KB x 2 B: the large schedule
    for sample in (False, True):
        V = 256 * 1024
        assert bench.early_exit_bytes(n, 15, V, es, sample) == _walk(n, LARGE[15], sample) * V * es


def test_early_exit_bytes_extremes():
    # every sequence rejects its first draft: the first wave of each (2 pairs here)
    assert bench.early_exit_bytes(np.zeros(4, int), 7, 10, 2, True) == 4 * 4 * 10 * 2
    # every draft accepted: the whole block, 2K + 1 rows (K + 1 greedy)
    assert bench.early_exit_bytes(np.full(3, 15), 15, 10, 2, True) == 3 * 31 * 10 * 2
    assert bench.early_exit_bytes(np.full(3, 15), 15, 10, 2, False) == 3 * 16 * 10 * 2
