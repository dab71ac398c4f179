"""The streaming sampler's split of rows x segments into one run per warp (host arithmetic).

Warp w streams units [floor(w T / W), floor((w + 1) T / W)); the per-row merge finds a row's
pieces from the runs alone, taking both floors of fp64 quotients (exact while the numerator is
below 2^53).  Checked here against integer division over the shapes the kernel sees: every unit
belongs to exactly one run, and the worker found for a unit is the one whose run holds it.
"""
import numpy as np


def _run_start(w, workers, total):
    return np.floor(np.float64(w * total) / np.float64(workers)).astype(np.int64)


def _worker_of(u, workers, total):
    return np.floor(np.float64((u + 1) * workers - 1) / np.float64(total)).astype(np.int64)


def test_fp64_floors_match_integer_division():
    rng = np.random.default_rng(0)
    cases = [(256, 128, 592 * 8), (256, 256, 444 * 8), (3, 1, 8), (1024, 512, 740 * 8),
             (1000, 7, 296 * 8), (1, 128, 16)]
    cases += [(int(rng.integers(1, 1025)), int(rng.integers(1, 513)), 8 * int(rng.integers(1, 1185)))
              for _ in range(40)]
    for rows, segs, workers in cases:
        total = rows * segs
        workers = min(workers, 8 * -(-total // 8))  # the launch clamps the grid to cdiv(units, 8)
        w = np.arange(workers + 1, dtype=np.int64)
        assert np.array_equal(_run_start(w, workers, total), (w * total) // workers)
        u = np.arange(total, dtype=np.int64)
        wu = _worker_of(u, workers, total)
        assert np.array_equal(wu, ((u + 1) * workers - 1) // total)
        starts = (np.arange(workers + 1, dtype=np.int64) * total) // workers
        assert np.all(starts[wu] <= u) and np.all(u < starts[wu + 1])


def test_row_pieces_cover_each_row_once():
    for rows, segs, workers in [(256, 128, 4736), (5, 10, 64), (3, 1, 8), (64, 13, 200)]:
        total = rows * segs
        workers = min(workers, 8 * -(-total // 8))
        starts = (np.arange(workers + 1, dtype=np.int64) * total) // workers
        for row in range(rows):
            r0 = row * segs
            w_lo, w_hi = _worker_of(np.int64(r0), workers, total), _worker_of(np.int64(r0 + segs - 1), workers, total)
            slots = [0]
            for k in range(1, int(w_hi - w_lo) + 1):
                a = int(_run_start(w_lo + k, workers, total))
                if w_lo + k < w_hi and a == int(_run_start(w_lo + k + 1, workers, total)):
                    continue  # empty run
                slots.append(a - r0)
            # the pieces tile the row: consecutive starts, each one a run start or the row start
            assert slots == sorted(set(slots)) and all(0 <= s < segs for s in slots)
            ends = slots[1:] + [segs]
            assert sum(e - s for s, e in zip(slots, ends)) == segs
            for s in slots[1:]:
                assert r0 + s in set(starts.tolist())
