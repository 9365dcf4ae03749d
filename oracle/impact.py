"""Row-impact scores -- TEST INFRASTRUCTURE ONLY.

A plain float64 restatement of the row-impact score of the hyper.ai summary
of the paper, section "方法" (Method), the paragraph on the spatial
distribution of errors: errors of equal size in different key rows reach the
readout with different weighting factors, derived from the transition matrix
and the query; a row's impact score is the expectation of the squared
weighting factor over calibration tokens.  The paragraph on key-row-aware
dual-axis fitting then uses the impact in the row factors and in the fit's
weights.  Only the tests may import this module.

Readings where the pages give no formula:
  * the weighting factor of key row i is the factor through which an error in
    that row of the stored state reaches the next readout: with the step's
    transition A = (I - beta k k^T) D (D = diag of the gates), the readout
    error is q^T A E, so for E = e_i eps^T the factor is (A^T q)_i =
    g_i (q_i - beta k_i (k . q));
  * the score is its mean square over the calibration (request, token)
    inputs, and the plan's weight is w_i = sqrt(score_i), so that the column
    fit's weight w_i^2 is the score itself.
"""

from __future__ import annotations

import numpy as np


def score_sum(q, k, beta, gate, gate_kind):
    """Sum over inputs of ((A^T q)_i)^2: q, k [n][H][d], beta [n][H], gate [n][H] or [n][H][d]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    beta = np.asarray(beta, np.float64)
    gate = np.asarray(gate, np.float64)
    n, H, d = q.shape
    out = np.zeros((H, d), np.float64)
    for h in range(H):
        for r in range(n):
            kq = 0.0
            for i in range(d):
                kq += k[r, h, i] * q[r, h, i]
            for i in range(d):
                g = gate[r, h, i] if gate_kind else gate[r, h]
                om = g * (q[r, h, i] - beta[r, h] * k[r, h, i] * kq)
                out[h, i] += om * om
    return out


def impact_weights(sums, count):
    """w = sqrt(sum / count), rounded to float32."""
    s = np.asarray(sums, np.float64)
    if count <= 0 or np.any(~np.isfinite(s)) or np.any(s <= 0):
        raise ValueError("scores must be finite and > 0, count > 0")
    return np.sqrt(s / count).astype(np.float32)
