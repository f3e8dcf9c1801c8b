"""Host-side helpers of bench.py (no GPU): the per-replay timing summary and
the seeded row sample of the prefill's oracle baseline."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_replay_stats_median_and_outlier():
    st = bench.replay_stats([1.0, 1.1, 0.9, 5.0, 1.0])
    assert st["median"] == 1.0
    assert st["min"] == 0.9 and st["max"] == 5.0 and st["n"] == 5
    assert abs(st["mean"] - 1.8) < 1e-12
    assert st["p90"] == 5.0                      # ceil(0.9 * 5) = 5th of 5
    st = bench.replay_stats([float(i) for i in range(1, 21)])
    assert st["median"] == 10.5 and st["p90"] == 18.0


def test_prefill_sample_rows():
    rows = bench.prefill_sample_rows(16384)
    assert len(rows) == 256 and len(set(rows)) == 256
    assert {0, 2047, 2048, 16383} <= set(rows)
    assert rows == sorted(rows) and rows[0] == 0 and rows[-1] == 16383
    assert rows == bench.prefill_sample_rows(16384)          # seeded
