"""The library's host-side allocation calls against the oracle (no GPU needed).

stepq_lifetime_weight and stepq_allocate_bits do no device work, so they run
here: the widths must equal the oracle's exactly (integer decisions from the
same float64 inputs), and bad arguments must be refused before anything is
written.
"""

import numpy as np
import pytest

from oracle import allocation as A


@pytest.fixture(scope="module")
def S():
    from quantized_delta_rule_decode_b200 import build as B
    B.build()
    import quantized_delta_rule_decode_b200 as S
    S.load_library()
    return S


CASES = [(1, 6, 0), (2, 6, 1), (7, 8, 2), (33, 4, 1), (257, 6, 3), (500, 8, 5), (4096, 6, 20)]


@pytest.mark.parametrize("n,budget,n_piv", CASES)
@pytest.mark.parametrize("shape", ["falling", "any", "ties"])
def test_allocate_bits_equals_the_oracle(S, n, budget, n_piv, shape):
    rng = np.random.default_rng(n * 7 + budget)
    L = rng.lognormal(0.0, 1.0, n)
    D = rng.lognormal(0.0, 1.0, (n, 3))
    if shape == "falling":
        D = -np.sort(-D, axis=1)
    elif shape == "ties":
        # few distinct values: exact ties in risks and in sums
        L = rng.integers(1, 3, n).astype(np.float64)
        D = np.array([[4.0, 2.0, 1.0], [3.0, 2.0, 1.0], [2.0, 2.0, 2.0]])[rng.integers(0, 3, n)]
    got = S.stepq_allocate_bits(L, D, budget, n_piv)
    want = A.allocate_bits(L, D, budget, n_piv)
    assert np.array_equal(got, want)


def test_lifetime_weight_equals_the_oracle(S):
    rng = np.random.default_rng(3)
    for shape in [(5, 4, 1), (3, 7, 2), (64, 32, 1)]:
        g = rng.uniform(0.05, 0.9995, shape).astype(np.float32)
        assert np.allclose(S.stepq_lifetime_weight(g), A.lifetime_weight(g), rtol=1e-14, atol=0)


def test_bad_arguments_are_refused(S):
    L, D = np.ones(4), np.ones((4, 3))
    for args in [(L, D, 5, 0), (L, D, 6, 5), (L, D, 6, -1), (-L, D, 6, 0), (L, -D, 6, 0),
                 (L * np.inf, D, 6, 0), (L, D * np.nan, 6, 0)]:
        with pytest.raises(S.StepqError):
            S.stepq_allocate_bits(*args)
    for g in [np.ones((2, 3, 1), np.float32), np.zeros((2, 3, 1), np.float32),
              np.full((2, 3, 1), np.nan, np.float32)]:
        with pytest.raises(S.StepqError):
            S.stepq_lifetime_weight(g)
