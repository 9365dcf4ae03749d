"""GPU decode step vs the oracle, through the C ABI.

One step: read packed state -> reconstruct -> gated Delta update -> readout
y = X^T q (before requantising) -> refit scales -> pack back (rcap.io post,
decode-step pseudocode; hyper.ai summary, "Method").  Both sides start from
the same packed state (packed by the oracle, copied to the device).

Tolerances:
  * y: relative L2 <= 1e-5 per step;
  * state: <= 0.1% of codes differ, by 1 only outside a re-scaled column;
    row factors / column scales differ in <= 0.1% of rows / columns.
The kernels meet the state contract with no difference at all (the tests
assert identical bytes), because delta, X and the column objective are
evaluated in the oracle's order.
"""

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import workload as W
from gpu_harness import (Pair, StepDiff, compare_pack, dev, lib, new_stats, pool_to_host, rel_l2,
                         rel_l2_worst_head, step_tensors)

pytestmark = pytest.mark.gpu


def _oracle_step(pair, pool_bytes, slots, si, rr, hh):
    """Oracle step of the chosen (request, head) pairs, in place on pool_bytes."""
    cfg = pair.cfg
    y = np.zeros((len(rr), cfg.d), np.float32)

    def one(t):
        r, h = rr[t], hh[t]
        off, nb = pair.ora.head_layout(h)
        base = slots[r] * pair.slot_bytes + off
        blob = pool_bytes[base:base + nb].copy()
        g = si.gate[r, h]
        yy, _, _ = pair.ora.step_head(h, blob, si.q[r, h], si.k[r, h], si.v[r, h], si.beta[r, h], g)
        pool_bytes[base:base + nb] = blob
        y[t] = yy

    with ThreadPoolExecutor(8) as ex:
        list(ex.map(one, range(len(rr))))
    return y


def _run_case(name, mode=W.MODE_STEPQUANT, ub=None, R=None, steps=1, two_streams=True, pivots=True):
    import torch
    cfg = W.CONFIGS[name]
    pair = Pair(cfg, mode=mode, uniform_bits=ub, pivots=pivots)
    S = lib()
    R = R or cfg.requests
    reqs = list(range(R))
    slots = W.slot_indices(cfg)[:R] if cfg.permute_slots else np.arange(R, dtype=np.int32)
    nslots = cfg.pool_slots if cfg.permute_slots else R
    X0 = W.initial_state(cfg, reqs)
    o = pair.ora.new_pool(nslots)
    assert pair.ora.pack(o, slots, X0) == 0
    pool = pair.gpu_pool(nslots)
    pool.buf.copy_(torch.from_numpy(o))
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")
    y = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream() if two_streams else None
    rr = [r for r in range(R) for _ in range(cfg.heads)]
    hh = [h for _ in range(R) for h in range(cfg.heads)]
    for step in range(steps):
        si = W.step_inputs(cfg, step, pair.pin, reqs)
        t = step_tensors(cfg, si)
        S.stepq_decode_step(pair.gpu, pool, dev(slots), t["q"], t["k"], t["v"], t["beta"], t["gate"],
                            y, ws, None, side)
        torch.cuda.synchronize()
        g = pool_to_host(pool)
        before = o.copy()
        yo = _oracle_step(pair, o, slots, si, rr, hh).reshape(R, cfg.heads, cfg.d)
        assert rel_l2(y.cpu().numpy(), yo) <= 1e-5
        assert rel_l2_worst_head(y.cpu().numpy(), yo) <= 1e-5
        diff = StepDiff()
        for r in range(R):
            for h in range(cfg.heads):
                diff.add(pair, h, pair.head_blob(g, slots[r], h), pair.head_blob(o, slots[r], h), None)
        diff.check(1e-3)
        # the readout hands the fit kernel a delta formed in the plain
        # definition's order, so the requantised state is identical
        assert diff.codes_diff == 0 and diff.rho_diff == 0 and diff.c_diff == 0
        assert np.array_equal(g, o)
        # keep both sides on the oracle's state for the next step
        pool.buf.copy_(torch.from_numpy(o))
        assert not np.array_equal(before, o)
    assert S.stepq_get_status(pool) == 0
    return pair


def test_step_tiny_16_steps():
    _run_case("tiny", steps=16)


def test_step_tiny_uniform6():
    _run_case("tiny", mode=W.MODE_UNIFORM, ub=6, steps=4)


def test_step_gdn():
    _run_case("gdn", R=6, steps=2)


def test_step_kda_permuted_slots():
    _run_case("kda", R=4, steps=2)


def test_step_pool_4bit():
    _run_case("pool", R=3)


def test_step_rollout_uniform8_single_stream():
    _run_case("rollout", mode=W.MODE_UNIFORM, ub=8, R=3, two_streams=False)


def test_step_kda_temporal_only():
    """Ablation: per-key-row widths and pivots, per-row scales only (no column fit)."""
    _run_case("kda", mode=W.MODE_UNIFORM, R=2, steps=2)


def test_step_kda_spatial_only():
    """Ablation: the dual-axis fit on uniform 6-bit key rows, no pivots."""
    _run_case("kda", mode=W.MODE_STEPQUANT, ub=6, R=2, steps=2)


def test_step_gdn_nopivot():
    """Ablation: the plan's widths with its FP16 pivot head quantised instead."""
    pair = _run_case("gdn", R=4, steps=2, pivots=False)
    assert not np.any(pair.pin.bits == 16)


def test_step_kda_nopivot():
    pair = _run_case("kda", R=2, steps=2, pivots=False)
    assert not np.any(pair.pin.bits == 16)


def test_two_streams_equal_one_stream_and_split_calls():
    """decode_step on two streams == on one stream == readout + fitpack called separately."""
    import torch
    cfg = W.CONFIGS["gdn"]
    pair = Pair(cfg)
    S = lib()
    R = 8
    X0 = W.initial_state(cfg, range(R))
    slots = dev(np.arange(R, dtype=np.int32))
    si = W.step_inputs(cfg, 0, pair.pin, range(R))
    t = step_tensors(cfg, si)
    outs = []
    for mode in ("two", "one", "split"):
        pool = pair.gpu_pool(R)
        S.stepq_pack(pair.gpu, pool, slots, dev(X0))
        ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")
        y = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
        if mode == "two":
            S.stepq_decode_step(pair.gpu, pool, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws,
                                None, torch.cuda.Stream())
        elif mode == "one":
            S.stepq_decode_step(pair.gpu, pool, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws)
        else:
            S.stepq_decode_readout(pair.gpu, pool, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws)
            S.stepq_decode_fitpack(pair.gpu, pool, slots, t["k"], t["gate"], ws)
        torch.cuda.synchronize()
        outs.append((y.cpu().numpy(), pool_to_host(pool)))
    for y, b in outs[1:]:
        assert np.array_equal(y, outs[0][0]) and np.array_equal(b, outs[0][1])


def test_unit_gate_zero_beta_keeps_reconstruction():
    """g = 1, beta = 0: X = S_prev exactly, so y = S_prev^T q and the refit state
    reconstructs S_prev to within half a quantisation step per entry."""
    import torch
    cfg = W.CONFIGS["tiny"]
    pair = Pair(cfg)
    S = lib()
    X0 = W.initial_state(cfg)
    slots = np.zeros(1, np.int32)
    o = pair.ora.new_pool(1)
    pair.ora.pack(o, slots, X0)
    Sprev, _ = pair.ora.unpack(o, slots)
    pool = pair.gpu_pool(1)
    pool.buf.copy_(torch.from_numpy(o))
    si = W.step_inputs(cfg, 0, pair.pin)
    si.beta[:] = 0.0
    si.gate[:] = 1.0
    t = step_tensors(cfg, si)
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, 1), dtype=torch.uint8, device="cuda")
    y = torch.empty((1, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
    S.stepq_decode_step(pair.gpu, pool, dev(slots), t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws)
    yref = np.einsum("hij,hi->hj", Sprev[0].astype(np.float64), si.q[0].astype(np.float64))
    assert rel_l2(y.cpu().numpy()[0], yref) <= 1e-6
    g = pool_to_host(pool)
    o2 = o.copy()
    _oracle_step(pair, o2, slots, si, [0] * cfg.heads, list(range(cfg.heads)))
    stats = new_stats()
    for h in range(cfg.heads):
        # identical X (= S_prev) on both sides -> the pack contract applies
        compare_pack(pair, h, pair.head_blob(g, 0, h), pair.head_blob(o2, 0, h), Sprev[0, h], stats)


@pytest.mark.parametrize("name", ["kda", "pool"])
def test_chunked_step_equals_one_launch_of_each_half(name):
    """A batch larger than the chunk budget (kda: 106 MB of packed state, pool:
    310 MB) is stepped chunk by chunk; its readout and state must be exactly
    those of one readout launch and one fit launch over the whole batch."""
    import torch
    cfg = W.CONFIGS[name]
    pair = Pair(cfg)
    S = lib()
    R = cfg.requests
    slots = dev(W.slot_indices(cfg))
    X = torch.randn((R, cfg.heads, cfg.d, cfg.d), dtype=torch.float32, device="cuda")
    X *= torch.exp(torch.randn((R, cfg.heads, cfg.d, 1), device="cuda"))
    si = W.step_inputs(cfg, 0, pair.pin)
    t = step_tensors(cfg, si)
    outs = []
    for how in ("chunked", "whole"):
        pool = pair.gpu_pool(cfg.pool_slots)
        S.stepq_pack(pair.gpu, pool, slots, X)
        ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")
        y = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
        if how == "chunked":
            S.stepq_decode_step(pair.gpu, pool, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws,
                                None, torch.cuda.Stream())
        else:
            S.stepq_decode_readout(pair.gpu, pool, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws)
            S.stepq_decode_fitpack(pair.gpu, pool, slots, t["k"], t["gate"], ws)
        torch.cuda.synchronize()
        outs.append((y.cpu().numpy(), pool_to_host(pool)))
        assert S.stepq_get_status(pool) == 0
        del pool, ws, y
    assert np.array_equal(outs[0][0], outs[1][0])
    assert np.array_equal(outs[0][1], outs[1][1])
