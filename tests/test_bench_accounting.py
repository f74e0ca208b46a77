"""Host-side accounting of bench.py: the bytes an early-exit call streams.

The waves read row pairs [0, 1), [1, 3), [3, 7), [7, 15), ... cut at K, the last adding the
bonus row, and each wave reads only the sequences that accepted every draft before it. The
schedules below are written out by hand for K = 0, 1, 2, 7 and 15 and walked sequence by
sequence, independently of the helper's own loop.
"""

import numpy as np

import bench

SCHEDULES = {
    0: [(0, 0)],
    1: [(0, 1)],
    2: [(0, 1), (1, 2)],
    7: [(0, 1), (1, 3), (3, 7)],
    15: [(0, 1), (1, 3), (3, 7), (7, 15)],
}


def _walk(n_accepted, K, sample):
    rows = 0
    waves = SCHEDULES[K]
    for j in n_accepted:
        for w, (lo, hi) in enumerate(waves):
            if j < lo:  # stopped in an earlier wave: nothing more is read
                break
            rows += (hi - lo) * (2 if sample else 1)
            if w == len(waves) - 1:
                rows += 1  # the bonus row
    return rows


def test_early_exit_bytes_follow_the_wave_schedule():
    rng = np.random.default_rng(0)
    for K in SCHEDULES:
        n = rng.integers(0, K + 1, size=200)
        for sample in (False, True):
            V, es = 1000, 2
            assert bench.early_exit_bytes(n, K, V, es, sample) == _walk(n, K, sample) * V * es


def test_early_exit_bytes_extremes():
    # every sequence rejects its first draft: one row pair each (one row when greedy)
    assert bench.early_exit_bytes(np.zeros(4, int), 7, 10, 2, True) == 4 * 2 * 10 * 2
    # every draft accepted: the whole block, 2K + 1 rows (K + 1 greedy)
    assert bench.early_exit_bytes(np.full(3, 15), 15, 10, 2, True) == 3 * 31 * 10 * 2
    assert bench.early_exit_bytes(np.full(3, 15), 15, 10, 2, False) == 3 * 16 * 10 * 2
