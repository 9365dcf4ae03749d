"""The oracle's lifetime-aware bit allocation, pinned to things other than itself.

Pages: hyper.ai summary, section "Method" (Lifetime-Aware Bit Allocation);
rcap.io post, "Temporal".  Pins:
  * the widths: exhaustive search over every allocation of small unit sets
    (the exact minimum of the lifetime-weighted distortion under the budget),
    pivots = the largest risks, the stated tie rule on exactly equal sums;
  * the lifetime weight: the geometric series in closed form, 1 / (1 - g)
    for a constant gate g, and the geometric mean of a unit's gates;
  * the distortion: zero for a zero state, the FP16 rounding error of a pivot
    plan from numpy's own binary16 conversion, head sums equal to the sums of
    the key-row units of the same quantisation.
"""

import itertools

import numpy as np
import pytest

import oracle
import workload as W
from oracle import allocation as A


def brute_force(L, D, budget, n_pivots):
    n = len(L)
    piv = set(A.pivot_order(L, D, budget)[:n_pivots])
    rest = [u for u in range(n) if u not in piv]
    best, best_bits = None, None
    for combo in itertools.product(range(3), repeat=len(rest)):
        if sum(4 + 2 * o for o in combo) > budget * len(rest):
            continue
        val = sum(float(L[u]) * float(D[u][o]) for u, o in zip(rest, combo))
        if best is None or val < best:
            best, best_bits = val, combo
    bits = np.full(n, 16, np.uint8)
    for u, o in zip(rest, best_bits or ()):
        bits[u] = 4 + 2 * o
    return best if best is not None else 0.0, bits


@pytest.mark.parametrize("seed", range(40))
def test_allocation_is_the_exact_minimum(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 8))
    budget = int(rng.choice([4, 6, 8]))
    n_piv = int(rng.integers(0, min(3, n) + 1))
    L = rng.lognormal(0.0, 1.0, n)
    D = rng.lognormal(0.0, 1.0, (n, 3))
    if seed % 2 == 0:
        D = -np.sort(-D, axis=1)          # distortion falling with width (the usual case)
    bits = A.allocate_bits(L, D, budget, n_piv)
    val, _ = brute_force(L, D, budget, n_piv)
    got = A.objective(L, D, bits)
    assert got <= val * (1 + 1e-12) + 1e-300
    rest = bits[bits != 16]
    assert int(np.sum(rest, dtype=np.int64)) <= budget * rest.size
    assert set(np.nonzero(bits == 16)[0]) == set(A.pivot_order(L, D, budget)[:n_piv])


def test_pivots_are_the_largest_risks_ties_to_lower_index():
    L = np.array([1.0, 2.0, 1.0, 0.5])
    D = np.array([[4.0, 2, 1], [2.0, 1, 0.5], [4.0, 2, 1], [1.0, 1, 1]])
    # risk at 6 bits: 2, 2, 2, 0.5 -> units 0, 1 (ties to the lower index)
    bits = A.allocate_bits(L, D, 6, 2)
    assert list(np.nonzero(bits == 16)[0]) == [0, 1]


def test_pivot_risk_is_taken_at_the_budget_width():
    # the risk of a unit is its lifetime weight times its distortion at the
    # budget width; the three widths rank these units differently:
    #   at 4 bits 10, 10, 12 -> unit 2;  at 6 bits 5, 4, 3 -> unit 0;  at 8 bits 1, 3, 2 -> unit 1
    L = np.ones(3)
    D = np.array([[10.0, 5, 1], [10.0, 4, 3], [12.0, 3, 2]])
    assert list(np.nonzero(A.allocate_bits(L, D, 6, 1) == 16)[0]) == [0]
    assert list(np.nonzero(A.allocate_bits(L, D, 8, 1) == 16)[0]) == [1]
    assert list(np.nonzero(A.allocate_bits(L, D, 4, 1) == 16)[0]) == [2]


def test_equal_sums_give_the_earlier_unit_the_smaller_width():
    # two identical units, costs 3, 2, 1 (exact in binary): (4, 8), (6, 6) and
    # (8, 4) all sum to 4; the stated rule picks (4, 8)
    L = np.ones(2)
    D = np.array([[3.0, 2.0, 1.0], [3.0, 2.0, 1.0]])
    assert list(A.allocate_bits(L, D, 6, 0)) == [4, 8]


def test_budget_four_is_all_four_bits():
    rng = np.random.default_rng(5)
    L, D = rng.lognormal(size=9), rng.lognormal(size=(9, 3))
    assert set(A.allocate_bits(L, D, 4, 0)) == {4}


def test_lifetime_weight_closed_forms():
    g = np.array([0.5, 0.9, 0.99, 0.999], np.float32)
    gates = np.broadcast_to(g[None, :, None], (7, 4, 1))
    L = A.lifetime_weight(gates)
    assert np.allclose(L, 1.0 / (1.0 - g.astype(np.float64)), rtol=1e-12)
    # two gates per unit: the mean log is the log of the geometric mean
    two = np.array([[[0.8, 0.98]]], np.float32)
    gm = np.sqrt(np.float64(np.float32(0.8)) * np.float64(np.float32(0.98)))
    assert np.isclose(A.lifetime_weight(two)[0], 1.0 / (1.0 - gm), rtol=1e-12)
    with pytest.raises(ValueError):
        A.lifetime_weight(np.array([[1.0]], np.float32))


def _plan(cfg, bits, mode=W.MODE_STEPQUANT, unit_kind=None):
    pin = W.make_plan(cfg)
    uk = cfg.unit_kind if unit_kind is None else unit_kind
    return oracle.Plan(cfg.d, cfg.d, cfg.heads, cfg.gate_kind, uk, mode, bits, pin.w)


def test_distortion_zero_state_is_zero():
    cfg = W.CONFIGS["tiny"]
    p = _plan(cfg, np.full(cfg.heads, 6, np.uint8))
    X = np.zeros((2, cfg.heads, cfg.d, cfg.d), np.float32)
    pool = p.new_pool(2)
    sl = np.array([1, 0], np.int32)
    assert p.pack(pool, sl, X) == 0
    dist, st = p.unit_distortion(pool, sl, X)
    assert st == 0 and np.all(dist == 0.0)


def test_distortion_of_a_pivot_plan_is_the_half_rounding_error():
    cfg = W.CONFIGS["tiny"]
    p = _plan(cfg, np.full(cfg.heads, 16, np.uint8))
    X = W.initial_state(cfg, [0])
    pool = p.new_pool(1)
    sl = np.array([0], np.int32)
    p.pack(pool, sl, X)
    dist, _ = p.unit_distortion(pool, sl, X)
    e = X.astype(np.float64) - X.astype(np.float16).astype(np.float64)
    want = (e * e).reshape(cfg.heads, -1).sum(axis=1)
    assert np.allclose(dist[0], want, rtol=1e-12, atol=0)


def test_head_distortion_is_the_sum_of_its_key_rows():
    cfg = W.CONFIGS["tiny"]
    X = W.initial_state(cfg, [0, 1])
    sl = np.array([0, 1], np.int32)
    ph = _plan(cfg, np.full(cfg.heads, 6, np.uint8), unit_kind=W.UNIT_HEAD)
    pr = _plan(cfg, np.full(cfg.heads * cfg.d, 6, np.uint8), unit_kind=W.UNIT_ROW)
    out = []
    for p in (ph, pr):
        pool = p.new_pool(2)
        p.pack(pool, sl, X)
        out.append((p.unit_distortion(pool, sl, X)[0], p.unpack(pool, sl)[0]))
    (dh, Sh), (dr, Sr) = out
    assert np.array_equal(Sh, Sr)            # one quantiser, two unit layouts
    for r in range(2):
        for h in range(cfg.heads):
            acc = 0.0
            for i in range(cfg.d):
                acc += dr[r, h * cfg.d + i]
            assert dh[r, h] == acc
    e = X.astype(np.float64) - Sh.astype(np.float64)
    assert np.allclose(dh, (e * e).reshape(2, cfg.heads, -1).sum(axis=2), rtol=1e-12)
