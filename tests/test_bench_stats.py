"""Statistics bench.py reports: the rank correlation of the lifetime study and
the per-launch busy time of kernels whose launches may overlap."""

import numpy as np

import bench


def test_spearman_hand_worked_with_ties():
    # ranks of b: 5 -> 1, 6 -> 2, the two 7s share (3 + 4) / 2 = 3.5, 8 -> 5;
    # against ranks 1..5 of a: cov = 4 + 1 + 0 + 2 + 1 = 8, var_a = 10,
    # var_b = 4 + 1 + 0.25 + 4 + 0.25 = 9.5, rho = 8 / sqrt(95)
    a = [1, 2, 3, 4, 5]
    b = [5, 6, 7, 8, 7]
    assert list(bench.rank_average(b)) == [1.0, 2.0, 3.5, 5.0, 3.5]
    assert abs(bench.spearman_rho(a, b) - 8 / np.sqrt(95)) < 1e-15


def test_spearman_without_ties_is_the_rank_difference_formula():
    # no ties: rho = 1 - 6 sum d^2 / (n (n^2 - 1)); d = rank differences
    a = [10.0, 20.0, 30.0, 40.0, 50.0, 60.0]
    b = [3.0, 1.0, 2.0, 6.0, 5.0, 4.0]      # ranks 3 1 2 6 5 4
    d2 = sum((i + 1 - r) ** 2 for i, r in enumerate([3, 1, 2, 6, 5, 4]))
    n = 6
    assert abs(bench.spearman_rho(a, b) - (1 - 6 * d2 / (n * (n * n - 1)))) < 1e-15
    assert bench.spearman_rho(a, a) == 1.0
    assert abs(bench.spearman_rho(a, a[::-1]) + 1.0) < 1e-15


def test_spearman_matches_scipy():
    from scipy import stats
    rng = np.random.default_rng(3)
    for _ in range(20):
        a = rng.integers(0, 30, 200).astype(float)   # many ties
        b = a + rng.normal(0, 10, 200)
        assert abs(bench.spearman_rho(a, b) - stats.spearmanr(a, b).statistic) < 1e-12


def test_busy_per_launch_disjoint_is_the_mean_duration():
    iv = [(0.0, 2.0), (5.0, 6.0), (10.0, 13.0)]
    assert bench.busy_per_launch(iv) == 2.0


def test_busy_per_launch_counts_overlap_once():
    # [0, 4] and [3, 7] cover [0, 7]; [7, 9] touches it; [12, 13] stands alone:
    # union 9 + 1 = 10 over 4 launches
    iv = [(3.0, 7.0), (0.0, 4.0), (12.0, 13.0), (7.0, 9.0)]
    assert bench.busy_per_launch(iv) == 2.5
    # one launch inside another adds nothing
    assert bench.busy_per_launch([(0.0, 10.0), (2.0, 3.0)]) == 5.0
    assert bench.busy_per_launch([]) == 0.0
