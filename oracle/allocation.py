"""Lifetime-aware bit allocation -- TEST INFRASTRUCTURE ONLY.

A plain restatement, in float64, of the offline step that chooses each state
unit's width before decoding starts:

  hyper.ai summary of the paper, section "方法" (Method), the paragraph on
  Lifetime-Aware Bit Allocation: per unit, the reconstruction distortion at
  each candidate width and the mean log retention; the error left after j
  updates decays exponentially, which gives a lifetime weight; under an
  average bit budget the widths minimise the lifetime-weighted distortion,
  and the riskiest units are kept in FP16 as sparse pivots.
  rcap.io post, the "Temporal" part (per-unit precisions from a candidate
  set under a budget; a small fraction of risky units in FP16) and the
  sentence placing allocation and pivot selection offline.

Only the tests may import this module.  It shares nothing with the library.

Readings where the pages give no formula:
  * mean log retention ell_u = the mean of log g over the unit's gates and
    the calibration steps; retention of an error after j updates exp(j ell_u);
    lifetime weight L_u = sum_{j >= 0} exp(j ell_u) = 1 / (1 - exp(ell_u)).
    Gates must lie in (0, 1).
  * distortion D_u(b) = squared reconstruction error of the unit's entries
    with the whole state quantised at width b (orc_unit_distortion), summed
    over the calibration states; candidate widths b in (4, 6, 8).
  * pivots: the n_pivots units of largest risk L_u * D_u(budget width), ties
    to the lower unit index.
  * widths of the other N units: minimise sum_u L_u * D_u(b_u) subject to
    sum_u b_u <= budget * N, exactly.  The minimum is taken by the recurrence
    V_u(k) = min over o in (0, 1, 2), o <= k, of c_u(o) + V_{u+1}(k - o),
    V_N(k) = 0, with c_u(o) = L_u * D_u(4 + 2 o) and k the number of 2-bit
    upgrades still allowed (K = N (budget - 4) / 2 at the start); on equal
    values the smaller o wins (compared in the order 0, 1, 2 with a strict <),
    and the widths are read forward from u = 0, k = K.
"""

from __future__ import annotations

import numpy as np

WIDTHS = (4, 6, 8)


def lifetime_weight(gates) -> np.ndarray:
    """gates [steps][units][rows] (or [steps][units]) -> L [units], float64."""
    g = np.asarray(gates, np.float64)
    if g.ndim == 2:
        g = g[:, :, None]
    if np.any(g <= 0.0) or np.any(g >= 1.0):
        raise ValueError("gates must lie in (0, 1)")
    steps, units, rows = g.shape
    out = np.zeros(units, np.float64)
    for u in range(units):
        acc = 0.0
        for t in range(steps):
            for r in range(rows):
                acc += np.log(g[t, u, r])
        ell = acc / (steps * rows)
        out[u] = 1.0 / (1.0 - np.exp(ell))
    return out


def pivot_order(L, D, budget):
    """Units by decreasing risk L_u * D_u(budget width), ties to the lower index."""
    col = WIDTHS.index(budget)
    risk = [L[u] * D[u][col] for u in range(len(L))]
    return sorted(range(len(L)), key=lambda u: (-risk[u], u))


def allocate_bits(L, D, budget: int, n_pivots: int) -> np.ndarray:
    """Widths (4, 6, 8, or 16 for a pivot) per unit, float64 arithmetic."""
    L = np.asarray(L, np.float64)
    D = np.asarray(D, np.float64)
    n = L.size
    if budget not in WIDTHS or not 0 <= n_pivots <= n or D.shape != (n, 3):
        raise ValueError("bad allocation arguments")
    bits = np.zeros(n, np.uint8)
    piv = set(pivot_order(L, D, budget)[:n_pivots])
    rest = [u for u in range(n) if u not in piv]
    for u in piv:
        bits[u] = 16
    N = len(rest)
    K = N * (budget - 4) // 2
    # backward recurrence over the remaining units, one vector over k per unit
    choice = np.zeros((N, K + 1), np.int8)
    nxt = np.zeros(K + 1, np.float64)
    for t in range(N - 1, -1, -1):
        u = rest[t]
        c = [L[u] * D[u][o] for o in range(3)]
        best = c[0] + nxt
        pick = np.zeros(K + 1, np.int8)
        for o in (1, 2):
            if K < o:
                continue
            cand = np.full(K + 1, np.inf)
            cand[o:] = c[o] + nxt[:K + 1 - o]
            better = cand < best
            best = np.where(better, cand, best)
            pick = np.where(better, np.int8(o), pick)
        choice[t] = pick
        nxt = best
    k = K
    for t in range(N):
        o = int(choice[t, k])
        bits[rest[t]] = WIDTHS[o]
        k -= o
    return bits


def objective(L, D, bits) -> float:
    """sum over non-pivot units of L_u * D_u(b_u), in ascending unit order."""
    tot = 0.0
    for u in range(len(L)):
        if bits[u] != 16:
            tot += float(L[u]) * float(D[u][WIDTHS.index(int(bits[u]))])
    return tot
