"""Host arithmetic of bench.py (no GPU): the per-row visible-key count that the
decode byte count and the CPU-baseline FLOPs use agrees with the oracle's mask
("Long Context: RoPE / YaRN / NTK / MLA", 10.1 sliding window and 10.2 sinks),
and its row sums with the work counter the FLOP totals use."""
import itertools
import types

import numpy as np
import pytest

import bench
import oracle
import workloads


@pytest.mark.parametrize("L,causal,W,S", [
    (L, c, W, S) for L, c, W, S in itertools.product((1, 7, 64), (True, False), (0, 1, 5, 64),
                                                     (0, 1, 3))
    if c or (W == 0 and S == 0)
])
def test_row_visible_matches_oracle_mask(L, causal, W, S):
    w = types.SimpleNamespace(L=L, causal=causal, window=W, sinks=S if W else 0)
    m = oracle.mask(L, causal, w.window, w.sinks)
    rows = [bench._row_visible(w, i) for i in range(L)]
    np.testing.assert_array_equal(rows, m.sum(axis=1))
    assert sum(rows) == workloads.visible_pairs(L, causal, w.window, w.sinks)


def test_job_tflops_is_whole_job_throughput():
    # 2 ranks x 4 steps x 1e12 FLOPs over the slowest rank's 25 ms
    assert bench.job_tflops(1e12, 2, 4, 25.0) == pytest.approx(2 * 4 * 1e12 / 0.025 / 1e12)
