"""The quantiser as its plain definition, in float64 -- TEST INFRASTRUCTURE ONLY.

A second reading of the requantisation of one head, written straight from
the definition with no binary32 evaluation order at all:

  hyper.ai summary of the paper, section "方法" (Method), the paragraph on
  key-row-aware dual-axis fitting: a per-key-row factor from the row's
  magnitude and its impact weight, per-column scales fitted by impact-weighted
  least squares, codes on the symmetric grid of the unit's width.
  rcap.io post, the decode-step pseudocode: r = sqrt(row magnitude) /
  sqrt(row impact weight); c = weighted least-squares fit with the squared
  impact weights; codes = quantize(X / (r c)).

Concrete form (the same readings as ``stepq_oracle.c``):

  m_i   = max_j |X_ij|                    (a NaN/Inf row is a zero row)
  rho_i = h(sqrt(m_i) / sqrt(w_i) * qmax_hi / qmax_i)     (uniform mode:
          h(m_i / qmax_i)); h = nearest binary16, ties to even, saturating,
          a positive value never rounded to zero
  M_j   = max_i |X_ij| / rho_i * qmax_hi / qmax_i        (active rows)
  c_a   = h(alpha_a M_j / qmax_hi), alpha_a = (100 - 5a) / 100, a = 0..7
  E_a   = sum_i w_i^2 (X_ij - rho_i c_a code_ia)^2,
          code_ia = clamp(rne(X_ij / (rho_i c_a)), +-qmax_i)
  best  = the first a of least E_a (ties to the larger alpha)

Every quotient, square root, product and sum is taken in float64 (numpy), in
plain ascending order; the only roundings that decide anything are the
binary16 roundings of the scales and the integer rounding of the codes,
which the definition itself asks for.  ``stepq_oracle.c`` instead fixes one
binary32 evaluation order for M_j and E_a; the tests compare the two
(``tests/test_oracle_fullsize_fit.py``), so that reading is pinned to this
one on full-size heads rather than only to itself.

Only the tests may import this module; it shares nothing with the library
and nothing with ``stepq_oracle.c`` (its own half rounding, by numpy's
float64 -> float16 conversion).
"""

from __future__ import annotations

import numpy as np

ALPHA = np.array([(100 - 5 * a) / 100.0 for a in range(8)], dtype=np.float64)
QMAX = {4: 7, 6: 31, 8: 127}
HALF_MAX = 65504.0


def half_bits(x) -> np.ndarray:
    """Nearest binary16 of float64 values (ties to even), saturating at
    +-65504, NaN -> 0; returned as uint16 bit patterns."""
    x = np.asarray(x, dtype=np.float64)
    x = np.where(np.isnan(x), 0.0, np.clip(x, -HALF_MAX, HALF_MAX))
    return x.astype(np.float16).view(np.uint16)


def half_value(bits) -> np.ndarray:
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def scale_bits(x) -> np.ndarray:
    """A positive scale as binary16: never rounds a positive value to zero."""
    x = np.asarray(x, dtype=np.float64)
    h = half_bits(x)
    return np.where((x > 0) & (h == 0), np.uint16(1), h).astype(np.uint16)


def row_factors(X, row_bits, w, mode=0):
    """rho (uint16 bits [dk]), active rows, non-finite flag.

    ``row_bits`` holds each key row's width (16 = FP16 pivot row)."""
    X = np.asarray(X, np.float64)
    dk = X.shape[0]
    rb = np.asarray(row_bits, np.int64)
    quant = rb != 16
    finite = np.all(np.isfinite(X), axis=1)
    m = np.where(finite, np.max(np.abs(np.where(np.isfinite(X), X, 0.0)), axis=1), 0.0)
    active = quant & (m > 0)
    qmax = np.array([QMAX.get(int(b), 0) for b in rb], np.float64)
    qhi = float(np.max(qmax[quant])) if np.any(quant) else 0.0
    rho = np.zeros(dk, np.uint16)
    if mode == 0:
        kap = np.where(quant, qhi / np.where(qmax > 0, qmax, 1.0), 0.0)
        r = np.sqrt(m) / np.sqrt(np.asarray(w, np.float64))
        rho[active] = scale_bits(r[active] * kap[active])
    else:
        rho[active] = scale_bits(m[active] / qmax[active])
    return rho, active, bool(np.any(quant & ~finite))


def column_maxima(X, rho_bits, active, row_bits):
    """M_j = max over active rows of |X_ij| / rho_i * qmax_hi / qmax_i."""
    X = np.asarray(X, np.float64)
    rb = np.asarray(row_bits, np.int64)
    qmax = np.array([QMAX.get(int(b), 0) for b in rb], np.float64)
    qhi = float(np.max(qmax[rb != 16])) if np.any(rb != 16) else 0.0
    rho = half_value(rho_bits)
    M = np.zeros(X.shape[1], np.float64)
    if np.any(active):
        z = np.abs(X[active]) / rho[active, None] * (qhi / qmax[active])[:, None]
        M = np.max(z, axis=0)
    return M, qhi


def candidates(M, qhi):
    """c_a = h(alpha_a M_j / qmax_hi) as uint16 bits [dv, 8]; zero where M_j = 0."""
    M = np.asarray(M, np.float64)
    c = scale_bits(ALPHA[None, :] * M[:, None] / qhi) if qhi > 0 else np.zeros((M.size, 8), np.uint16)
    c[M == 0] = 0
    return c


def codes_under(X, rho_bits, active, row_bits, c_bits_col):
    """clamp(rne(X_ij / (rho_i c_j)), +-qmax_i) for every entry, with one
    column scale per column (``c_bits_col`` [dv]); 0 on inactive rows and
    zero columns."""
    X = np.asarray(X, np.float64)
    rb = np.asarray(row_bits, np.int64)
    qmax = np.array([QMAX.get(int(b), 0) for b in rb], np.float64)
    P = half_value(rho_bits)[:, None] * half_value(c_bits_col)[None, :]
    ok = active[:, None] & (P > 0)
    t = np.where(ok, X / np.where(ok, P, 1.0), 0.0)
    q = np.clip(np.rint(t), -qmax[:, None], qmax[:, None])
    return np.where(ok, q, 0.0).astype(np.int16)


def objectives(X, rho_bits, active, row_bits, w, cand_bits):
    """E[j, a] = sum_i w_i^2 (X_ij - rho_i c_ja code_ija)^2 in float64 over
    the active rows, ascending i; also the per-term quantities a caller
    needs for error bounds: sum_i w_i^2 |e| |X| per (j, a)."""
    X = np.asarray(X, np.float64)
    dk, dv = X.shape
    w2 = np.asarray(w, np.float64) ** 2
    E = np.zeros((dv, 8), np.float64)
    C = np.zeros((dv, 8), np.float64)
    rho = half_value(rho_bits)
    for a in range(8):
        ca = half_value(cand_bits[:, a])
        code = codes_under(X, rho_bits, active, row_bits, cand_bits[:, a]).astype(np.float64)
        e = np.where(active[:, None], X - (rho[:, None] * ca[None, :]) * code, 0.0)
        E[:, a] = np.sum(w2[:, None] * e * e, axis=0)
        C[:, a] = np.sum(w2[:, None] * np.abs(e) * np.abs(X) * active[:, None], axis=0)
    return E, C


def argmin_first(E):
    """Index of the least value per row, the first one on ties (larger alpha)."""
    E = np.asarray(E)
    best = np.zeros(E.shape[0], np.int64)
    for a in range(1, E.shape[1]):
        best = np.where(E[:, a] < E[np.arange(E.shape[0]), best], a, best)
    return best


def quantize_head(X, row_bits, w, mode=0, head_pivot=False):
    """The whole requantisation of one head by the definition.

    Returns a dict with uint16 ``rho`` [dk], ``c`` [dv], int16 ``codes``
    [dk, dv], uint16 ``piv`` [dk, dv] (FP16 pivot rows / heads), ``best``,
    ``cand`` [dv, 8], float64 ``E`` [dv, 8] and ``M`` [dv], and the
    non-finite flag."""
    X = np.asarray(X, np.float64)
    dk, dv = X.shape
    rb = np.full(dk, 16, np.int64) if head_pivot else np.asarray(row_bits, np.int64)
    out = dict(rho=np.zeros(dk, np.uint16), c=np.zeros(dv, np.uint16),
               codes=np.zeros((dk, dv), np.int16), piv=np.zeros((dk, dv), np.uint16),
               best=np.zeros(dv, np.int64), cand=np.zeros((dv, 8), np.uint16),
               E=np.zeros((dv, 8)), M=np.zeros(dv), nonfinite=False)
    pivot_rows = rb == 16
    out["piv"][pivot_rows] = half_bits(X[pivot_rows])
    out["nonfinite"] = bool(np.any(~np.isfinite(X[pivot_rows])))
    if head_pivot:
        return out
    rho, active, bad = row_factors(X, rb, w, mode)
    out["rho"] = rho
    out["nonfinite"] |= bad
    Xa = np.where(np.isfinite(X), X, 0.0)
    if mode == 1:
        c = np.full(dv, 0x3C00, np.uint16)  # 1.0
    else:
        M, qhi = column_maxima(Xa, rho, active, rb)
        cand = candidates(M, qhi)
        E, _ = objectives(Xa, rho, active, rb, w, cand)
        best = argmin_first(E)
        c = np.where(M > 0, cand[np.arange(dv), best], 0).astype(np.uint16)
        out.update(M=M, cand=cand, E=E, best=best)
    out["c"] = c
    out["codes"] = codes_under(Xa, rho, active, rb, c)
    return out
