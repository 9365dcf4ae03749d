"""The oracle's row-impact scores, pinned to things other than itself.

hyper.ai summary, section "Method" (spatial distribution of errors; key-row-
aware dual-axis fitting).  Pins: the weighting factor equals (A^T q)_i for the
transition A = (I - beta k k^T) D built as a matrix and multiplied by numpy;
beta = 0 leaves g q; a key along the query with beta = 1 removes the query
(factor 0); a diagonal gate with equal entries equals the scalar gate; the
library's host weight call gives the same fp32 weights.
"""

import numpy as np
import pytest

from oracle import impact as I


def _inputs(seed, n=3, H=2, d=16, diag=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n, H, d)).astype(np.float32)
    k = rng.standard_normal((n, H, d)).astype(np.float32)
    k /= np.linalg.norm(k, axis=2, keepdims=True)
    beta = rng.uniform(0, 1, (n, H)).astype(np.float32)
    gate = rng.uniform(0.5, 1, (n, H, d) if diag else (n, H)).astype(np.float32)
    return q, k, beta, gate


@pytest.mark.parametrize("diag", [False, True])
def test_score_is_the_transition_applied_to_the_query(diag):
    q, k, beta, gate = _inputs(1, diag=diag)
    n, H, d = q.shape
    want = np.zeros((H, d))
    for r in range(n):
        for h in range(H):
            g = gate[r, h] if diag else np.full(d, gate[r, h])
            kk = k[r, h].astype(np.float64)[:, None]
            A = (np.eye(d) - np.float64(beta[r, h]) * (kk @ kk.T)) @ np.diag(g.astype(np.float64))
            om = A.T @ q[r, h].astype(np.float64)
            want[h] += om * om
    assert np.allclose(I.score_sum(q, k, beta, gate, int(diag)), want, rtol=1e-12, atol=0)


def test_special_cases():
    q, k, beta, gate = _inputs(2)
    s0 = I.score_sum(q, k, np.zeros_like(beta), gate, 0)
    want = ((gate[:, :, None].astype(np.float64) * q) ** 2).sum(axis=0)
    assert np.allclose(s0, want, rtol=1e-14, atol=0)
    # a key along the query with beta = 1: the update removes the query's direction
    k1 = q / np.linalg.norm(q.astype(np.float64), axis=2, keepdims=True)
    s1 = I.score_sum(q, k1, np.ones_like(beta), gate, 0)
    assert np.max(s1) < 1e-12 * np.max(s0)
    # equal diagonal gates = the scalar gate
    gd = np.repeat(gate[:, :, None], q.shape[2], axis=2)
    assert np.array_equal(I.score_sum(q, k, beta, gd, 1), I.score_sum(q, k, beta, gate, 0))


def test_weights_and_library_host_call():
    from quantized_delta_rule_decode_b200 import build as B
    B.build()
    import quantized_delta_rule_decode_b200 as S
    rng = np.random.default_rng(4)
    sums = rng.lognormal(0, 2, 500)
    w = I.impact_weights(sums, 37)
    assert np.allclose(w.astype(np.float64) ** 2 * 37, sums, rtol=2e-7)
    assert np.array_equal(S.stepq_impact_weights(sums, 37), w)
    for bad in (np.zeros(3), np.full(3, np.nan), -np.ones(3)):
        with pytest.raises(S.StepqError):
            S.stepq_impact_weights(bad, 5)
    with pytest.raises(S.StepqError):
        S.stepq_impact_weights(np.ones(3), 0)
