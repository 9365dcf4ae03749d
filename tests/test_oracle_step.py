"""Pins the oracle's gated Delta update and readout.

The equation (rcap.io post, decode-step pseudocode; hyper.ai summary, Method):
    X = D S + beta k (v^T - k^T D S),   y = X^T q   (readout before requantising)
with D = g I (scalar gate, GDN) or diag(g) (per-key-row gate, KDA).

Pins, none of which re-types the oracle's loops:
* g = 1, beta = 0 leaves the state unchanged, bit for bit;
* g = 1, beta = 1 and a unit key write v into the key direction: k^T X = v^T
  (exactly for k = e_i on integer data, to the fp32 rounding bound otherwise);
* the matrix form evaluated by numpy in float64 with matmul/outer, to within
  the fp32 rounding bound of the oracle's sums;
* a diagonal gate with all entries equal reproduces the scalar gate exactly;
* the fp32 baseline step is the same update applied in place.
"""

import numpy as np
import pytest

import workload as W

U = 2.0 ** -24


def _rand_head(rng, dk, dv, scale=1.0):
    S = (rng.standard_normal((dk, dv)) * scale).astype(np.float32)
    q = rng.standard_normal(dk).astype(np.float32)
    q /= np.float32(np.linalg.norm(q))
    k = rng.standard_normal(dk).astype(np.float32)
    k /= np.float32(np.linalg.norm(k))
    v = rng.standard_normal(dv).astype(np.float32)
    return S, q, k, v


@pytest.mark.parametrize("gate_kind", [0, 1])
def test_unit_gate_zero_beta_leaves_state(orc, gate_kind):
    rng = np.random.default_rng(1)
    for dk, dv in [(64, 64), (128, 128), (7, 5)]:
        S, q, k, v = _rand_head(rng, dk, dv, 3.0)
        gate = np.ones(dk if gate_kind else 1, np.float32)
        X, y = orc.delta_update(S, q, k, v, 0.0, gate, gate_kind)
        assert np.array_equal(X.view(np.uint32), S.view(np.uint32))
        ref = S.astype(np.float64).T @ q.astype(np.float64)
        bound = dk * U * (np.abs(S.astype(np.float64)).T @ np.abs(q.astype(np.float64))) * 1.01
        assert np.all(np.abs(y - ref) <= bound + 1e-30)


def test_delta_write_basis_key_exact(orc):
    """k = e_i, g = 1, beta = 1: row i of X becomes v, every other row is kept."""
    rng = np.random.default_rng(2)
    dk, dv = 16, 12
    S = rng.integers(-64, 64, size=(dk, dv)).astype(np.float32)
    v = rng.integers(-64, 64, size=dv).astype(np.float32)
    q = rng.standard_normal(dk).astype(np.float32)
    for i in [0, 5, dk - 1]:
        k = np.zeros(dk, np.float32)
        k[i] = 1.0
        X, _ = orc.delta_update(S, q, k, v, 1.0, np.ones(1, np.float32), 0)
        assert np.array_equal(X[i], v)
        keep = np.arange(dk) != i
        assert np.array_equal(X[keep], S[keep])


@pytest.mark.parametrize("gate_kind", [0, 1])
def test_delta_write_unit_key(orc, gate_kind):
    """g = 1, beta = 1, |k| = 1: k^T X = v^T within the fp32 rounding bound."""
    rng = np.random.default_rng(3)
    for dk, dv in [(64, 64), (128, 128)]:
        S, q, k, v = _rand_head(rng, dk, dv, 2.0)
        gate = np.ones(dk if gate_kind else 1, np.float32)
        X, _ = orc.delta_update(S, q, k, v, 1.0, gate, gate_kind)
        k64 = k.astype(np.float64)
        lhs = k64 @ X.astype(np.float64)
        # exact algebra gives v + (1 - |k|^2)(v - k^T S); |k|^2 differs from 1 by rounding
        kk = k64 @ k64
        ideal = v + (1.0 - kk) * (v - k64 @ S.astype(np.float64))
        absS = np.abs(k64) @ np.abs(S.astype(np.float64))
        bound = 4 * dk * U * (absS + np.abs(v) + np.abs(k64) @ np.abs(X.astype(np.float64)))
        assert np.all(np.abs(lhs - ideal) <= bound)
        assert np.max(np.abs(lhs - v)) < 1e-4


@pytest.mark.parametrize("gate_kind", [0, 1])
def test_matrix_form_float64(orc, gate_kind):
    rng = np.random.default_rng(4)
    for dk, dv in [(64, 64), (128, 128), (32, 48)]:
        S, q, k, v = _rand_head(rng, dk, dv, 5.0)
        gate = rng.uniform(0.5, 1.0, size=dk if gate_kind else 1).astype(np.float32)
        beta = np.float32(rng.uniform(0.1, 0.9))
        X, y = orc.delta_update(S, q, k, v, beta, gate, gate_kind)
        D = np.diag(gate.astype(np.float64)) if gate_kind else float(gate[0]) * np.eye(dk)
        S64, k64, v64, q64 = (a.astype(np.float64) for a in (S, k, v, q))
        DS = D @ S64
        X64 = DS + float(beta) * np.outer(k64, v64 - k64 @ DS)
        y64 = X64.T @ q64
        # first-order rounding bound of the oracle's fp32 evaluation
        u_abs = np.abs(k64) @ np.abs(DS)
        d_abs = float(beta) * (np.abs(v64) + u_abs) + float(beta) * dk * U * u_abs * 4
        bX = 4 * U * (np.abs(DS) + np.outer(np.abs(k64), d_abs)) + \
            np.outer(np.abs(k64), float(beta) * (dk + 2) * U * u_abs)
        assert np.all(np.abs(X - X64) <= bX * 1.5 + 1e-30)
        by = (dk + 2) * U * (np.abs(X64).T @ np.abs(q64)) + np.abs(q64) @ bX * 1.5
        assert np.all(np.abs(y - y64) <= by + 1e-30)


def test_uniform_diag_gate_equals_scalar(orc):
    rng = np.random.default_rng(5)
    S, q, k, v = _rand_head(rng, 64, 64, 1.0)
    g = np.float32(0.9)
    X0, y0 = orc.delta_update(S, q, k, v, 0.7, np.array([g]), 0)
    X1, y1 = orc.delta_update(S, q, k, v, 0.7, np.full(64, g, np.float32), 1)
    assert np.array_equal(X0, X1) and np.array_equal(y0, y1)


def test_fp32_step_is_update_in_place(orc):
    cfg = W.CONFIGS["tiny"]
    p = W.make_plan(cfg)
    S0 = W.initial_state(cfg)
    si = W.step_inputs(cfg, 0, p)
    S = S0.copy()
    y, st = orc.fp32_step(S, W.slot_indices(cfg), si.q, si.k, si.v, si.beta, si.gate, cfg.gate_kind)
    assert st == 0
    for h in range(cfg.heads):
        X, yy = orc.delta_update(S0[0, h], si.q[0, h], si.k[0, h], si.v[0, h], si.beta[0, h],
                                 si.gate[0, h], cfg.gate_kind)
        assert np.array_equal(S[0, h], X) and np.array_equal(y[0, h], yy)


def test_bad_slot_flagged(orc):
    cfg = W.CONFIGS["tiny"]
    p = W.make_plan(cfg)
    S = W.initial_state(cfg)
    si = W.step_inputs(cfg, 0, p)
    before = S.copy()
    y, st = orc.fp32_step(S, np.array([5], np.int32), si.q, si.k, si.v, si.beta, si.gate, 0)
    assert st & orc.STATUS_BAD_SLOT and np.array_equal(S, before)
