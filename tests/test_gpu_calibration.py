"""Lifetime-aware bit allocation on the GPU path vs the oracle.

hyper.ai summary, section "Method" (Lifetime-Aware Bit Allocation): per-unit
distortion at each width, a lifetime weight, widths under a budget, FP16
pivots.  The distortion kernel must match the oracle's float64 sums to
rounding (different summation order); the widths are integer decisions and
must match exactly unless two allocations are equal to within that rounding.
"""

import numpy as np
import pytest

import oracle
import workload as W
from gpu_harness import Pair, dev, lib, pool_to_host
from oracle import allocation as A

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,R", [("tiny", 1), ("gdn", 2), ("kda", 2)])
def test_unit_distortion_matches_oracle(name, R):
    import torch
    cfg = W.CONFIGS[name]
    pair = Pair(cfg)
    S = lib()
    slots = W.slot_indices(cfg)[:R] if cfg.permute_slots else np.arange(R, dtype=np.int32)
    nslots = cfg.pool_slots if cfg.permute_slots else R
    X = W.initial_state(cfg, list(range(R)))
    pool = pair.gpu_pool(nslots)
    Xd = dev(X)
    S.stepq_pack(pair.gpu, pool, dev(slots), Xd)
    o = pair.ora.new_pool(nslots)
    assert pair.ora.pack(o, slots, X) == 0
    assert np.array_equal(pool_to_host(pool), o)      # same packed state on both sides
    dist = S.stepq_unit_distortion(pair.gpu, pool, dev(slots), Xd)
    torch.cuda.synchronize()
    got = dist.cpu().numpy()
    want, st = pair.ora.unit_distortion(o, slots, X)
    assert st == 0
    assert got.shape == want.shape
    assert np.allclose(got, want, rtol=1e-11, atol=0)
    assert S.stepq_get_status(pool) == 0


@pytest.mark.parametrize("name", ["gdn", "kda"])
def test_unit_distortion_accumulates_on_device(name):
    """dist_sum += the distortion summed over requests, over two calls: the
    oracle's per-request values summed in float64 (rel 1e-11: the device
    adds in another order)."""
    import torch
    cfg = W.CONFIGS[name]
    pair = Pair(cfg)
    S = lib()
    R = 3
    slots = W.slot_indices(cfg)[:R] if cfg.permute_slots else np.arange(R, dtype=np.int32)
    nslots = cfg.pool_slots if cfg.permute_slots else R
    units = cfg.units
    total = torch.zeros(units, dtype=torch.float64, device="cuda")
    want = np.zeros(units, np.float64)
    for call in range(2):
        X = W.initial_state(cfg, [call * R + r for r in range(R)])
        pool = pair.gpu_pool(nslots)
        Xd = dev(X)
        S.stepq_pack(pair.gpu, pool, dev(slots), Xd)
        S.stepq_unit_distortion_accumulate(pair.gpu, pool, dev(slots), Xd, total)
        o = pair.ora.new_pool(nslots)
        assert pair.ora.pack(o, slots, X) == 0
        d, st = pair.ora.unit_distortion(o, slots, X)
        assert st == 0
        want += d.sum(axis=0)
        assert S.stepq_get_status(pool) == 0
    got = total.cpu().numpy()
    assert np.allclose(got, want, rtol=1e-11, atol=0)


def _gates(cfg, pin):
    g = np.asarray(pin.gate, np.float32)
    if cfg.unit_kind == W.UNIT_ROW:
        g = g.reshape(-1) if cfg.gate_kind == W.GATE_DIAG else np.repeat(g, cfg.d)
    else:
        g = g.reshape(cfg.heads, -1).mean(axis=1) if g.ndim == 2 else g
    return g[None, :, None]


def _oracle_dist(cfg, pin, states):
    units = cfg.units
    total = np.zeros((units, 3), np.float64)
    for col, b in enumerate(A.WIDTHS):
        p = oracle.Plan(cfg.d, cfg.d, cfg.heads, cfg.gate_kind, cfg.unit_kind, W.MODE_STEPQUANT,
                        np.full(units, b, np.uint8), pin.w)
        for X in states:
            n = X.shape[0]
            pool = p.new_pool(n)
            sl = np.arange(n, dtype=np.int32)
            assert p.pack(pool, sl, X) == 0
            d, st = p.unit_distortion(pool, sl, X)
            assert st == 0
            for r in range(n):
                total[:, col] += d[r]
    return total


@pytest.mark.parametrize("name", ["tiny", "kda"])
def test_calibration_matches_oracle(name):
    from quantized_delta_rule_decode_b200 import calibrate
    cfg = W.CONFIGS[name]
    pin = W.make_plan(cfg)
    states = [W.initial_state(cfg, [0, 1]), W.initial_state(cfg, [2])]
    gates = _gates(cfg, pin)
    n_piv = int(np.sum(pin.bits == 16))
    budget = cfg.budget
    bits, weight, dist = calibrate.calibrate_bits(cfg.d, cfg.d, cfg.heads, cfg.gate_kind,
                                                  cfg.unit_kind, pin.w, [dev(X) for X in states],
                                                  gates, budget, n_piv)
    dist_o = _oracle_dist(cfg, pin, states)
    weight_o = A.lifetime_weight(gates)
    assert np.allclose(dist, dist_o, rtol=1e-11, atol=0)
    assert np.allclose(weight, weight_o, rtol=1e-14, atol=0)
    bits_o = A.allocate_bits(weight_o, dist_o, budget, n_piv)
    if not np.array_equal(bits, bits_o):
        # only an allocation of equal value, to the rounding of the inputs
        a, b = A.objective(weight_o, dist_o, bits), A.objective(weight_o, dist_o, bits_o)
        assert abs(a - b) <= 1e-9 * b
    rest = bits[bits != 16]
    assert np.sum(rest, dtype=np.int64) <= budget * rest.size
    assert np.sum(bits == 16) == n_piv


@pytest.mark.parametrize("name", ["gdn", "kda", "tiny"])
def test_row_impact_matches_oracle(name):
    """Row-impact scores (hyper.ai, Method: the spatial paragraph): two
    accumulating calls over 3 requests each, against the oracle's float64 sums."""
    import torch

    from oracle import impact as I
    from gpu_harness import step_tensors
    cfg = W.CONFIGS[name]
    pin = W.make_plan(cfg)
    S = lib()
    reqs = [0, 1, 2]
    score = torch.zeros((cfg.heads, cfg.d), dtype=torch.float64, device="cuda")
    want = np.zeros((cfg.heads, cfg.d))
    for step in (0, 1):
        si = W.step_inputs(cfg, step, pin, reqs)
        t = step_tensors(cfg, si)
        S.stepq_row_impact(cfg.gate_kind, t["q"], t["k"], t["beta"], t["gate"], score)
        want += I.score_sum(si.q, si.k, si.beta, si.gate, cfg.gate_kind)
    torch.cuda.synchronize()
    assert np.allclose(score.cpu().numpy(), want, rtol=1e-12, atol=0)
    w = S.stepq_impact_weights(score.cpu().numpy(), 2 * len(reqs))
    assert np.allclose(w, I.impact_weights(want, 2 * len(reqs)).reshape(-1), rtol=1e-6, atol=0)
