"""Pins the oracle's binary32 column fit to the plain definition on full-size heads.

``stepq_oracle.c`` evaluates the column maximum M_j = max_i |X_ij / rho_i|
and the objective E_a = sum_i w_i^2 (X_ij - rho_i c_a code_ij)^2 in one
stated binary32 order (the quotient by rho_i as a product with its rounded
reciprocal; the objective in step units with four partial sums).  The pages
fix no order (rcap.io post, decode-step pseudocode: ``fit_weighted_lsq`` with
squared impact weights; hyper.ai summary, Method, dual-axis fitting), so the
order is a reading; these tests hold it to the definition itself, evaluated
in float64 with no order at all (``oracle/definition.py``), on d = 128 heads
of every full-size workload -- GDN heads of each width, KDA heads with mixed
row widths and FP16 pivot rows, the 4-bit pool, the rollout plan -- both on
the initial states and on the states after one decode step:

* row factors and the 8 candidate scales equal the definition's, except where
  the exact value lies within 2^-20 of a binary16 rounding midpoint (a few
  binary32 roundings can move it across);
* each candidate's objective is within the binary32 evaluation bound of the
  float64 one;
* the chosen candidate is the definition's argmin (ties to the larger alpha),
  except where the two objectives lie within the sum of their bounds; such
  near ties are counted and must stay under 0.1% of columns;
* codes equal clamp(rne(X / (rho c)), +-qmax) except within 2^-22 of a tie;
* end to end (definition vs oracle, each with its own scales), at most 0.1%
  of the codes differ, and outside columns whose scale differs only by 1.
"""

import numpy as np
import pytest

import workload as W
from oracle import definition as D

U = 2.0 ** -24
HEADS_PER_WORKLOAD = 64


def half_mid_distance(v):
    """Relative distance of positive float64 values to the nearest binary16
    rounding midpoint (normal and subnormal range)."""
    v = np.asarray(v, np.float64)
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -30)))
    g = np.where(v < 2.0 ** -14, 2.0 ** -24, 2.0 ** (e - 10))
    t = v / g
    return np.abs(t - np.floor(t) - 0.5) * g / np.maximum(v, 1e-300)


def _row_bits(cfg, pin, h):
    if cfg.unit_kind == W.UNIT_ROW:
        return pin.bits[h * cfg.d:(h + 1) * cfg.d].astype(np.int64)
    return np.full(cfg.d, int(pin.bits[h]), np.int64)


def _cases(orc, name):
    """(plan, head, X, row_bits, w) for HEADS_PER_WORKLOAD quantised heads of
    the workload, each on S0 and on the state after one oracle decode step."""
    cfg = W.CONFIGS[name]
    pin = W.make_plan(cfg)
    ora = orc.Plan(cfg.d, cfg.d, cfg.heads, cfg.gate_kind, cfg.unit_kind, 0, pin.bits, pin.w)
    heads = [h for h in range(cfg.heads)
             if not (cfg.unit_kind == W.UNIT_HEAD and pin.bits[h] == 16)]
    pairs = [(r, h) for r in range((HEADS_PER_WORKLOAD + len(heads) - 1) // len(heads))
             for h in heads][:HEADS_PER_WORKLOAD]
    for r, h in pairs:
        X0 = W.initial_state(cfg, [r], [h])[0, 0]
        rb = _row_bits(cfg, pin, h)
        yield ora, h, X0, rb, pin.w[h]
        blob, st = ora.quantize_head(h, X0)
        assert st == 0
        si = W.step_inputs(cfg, 0, pin, requests=[r], heads=[h])
        g = si.gate[0, 0]
        _, X1, st = ora.step_head(h, blob, si.q[0, 0], si.k[0, 0], si.v[0, 0], si.beta[0, 0], g)
        assert st == 0
        yield ora, h, X1, rb, pin.w[h]


def _check(ora, h, X, rb, w, st):
    dk, dv = X.shape
    Xd = X.astype(np.float64)
    blob, status, E_o, cand_o, best_o = ora.quantize_head(h, X, diag=True)
    assert status == 0
    codes_o, piv_o, rho_o, c_o = ora.unpack_codes(h, blob)
    qmax = np.array([D.QMAX.get(int(b), 0) for b in rb], np.float64)
    quant = rb != 16
    qhi = float(qmax[quant].max())

    # ---- row factors: h(sqrt(m)/sqrt(w) * qmax_hi/qmax_i) ----
    rho_d, act_d, _ = D.row_factors(Xd, rb, w)
    m = np.max(np.abs(Xd), axis=1)
    pre = np.sqrt(m) / np.sqrt(w.astype(np.float64)) * np.where(quant, qhi / np.maximum(qmax, 1), 0)
    act = quant & (rho_o > 0)
    assert np.array_equal(act, act_d)
    edge = act & (half_mid_distance(np.where(act, pre, 1.0)) <= 2.0 ** -20)
    st["rows"] += int(act.sum())
    st["rho_boundary"] += int(edge.sum())
    assert np.array_equal(rho_o[act & ~edge], rho_d[act & ~edge])
    assert np.all(np.abs(rho_o[edge].astype(np.int64) - rho_d[edge].astype(np.int64)) <= 1)

    # ---- M_j and the candidates, given the oracle's row factors ----
    M_d, _ = D.column_maxima(Xd, rho_o, act, rb)
    cand_d = D.candidates(M_d, qhi)
    live = M_d > 0
    pre_c = D.ALPHA[None, :] * M_d[:, None] / qhi
    cedge = live[:, None] & (half_mid_distance(np.where(live[:, None], pre_c, 1.0)) <= 2.0 ** -20)
    st["cands"] += int(live.sum()) * 8
    st["cand_boundary"] += int(cedge.sum())
    ok = live[:, None] & ~cedge
    assert np.array_equal(cand_o[ok], cand_d[ok])
    assert np.all(np.abs(cand_o[cedge].astype(np.int64) - cand_d[cedge].astype(np.int64)) <= 1)
    assert np.all(c_o[~live] == 0)

    # ---- objectives under the oracle's candidates, within the binary32 bound ----
    E_d, C_d = D.objectives(Xd, rho_o, act, rb, w, cand_o)
    n_act = int(act.sum())
    bound = (n_act + 12) * U * E_d + 8 * U * C_d
    Eo = E_o.astype(np.float64)
    assert np.all(np.abs(Eo[live] - E_d[live]) <= bound[live])

    # ---- argmin (ties to the larger alpha) ----
    best_d = D.argmin_first(E_d)
    cols = np.flatnonzero(live)
    st["columns"] += cols.size
    for j in cols:
        srt = np.sort(E_d[j])
        b_top = bound[j][np.argsort(E_d[j])]
        if srt[1] - srt[0] <= b_top[0] + b_top[1]:
            st["close_pairs"] += 1          # the two best within the bound
        if best_o[j] != best_d[j]:
            a, b = int(best_o[j]), int(best_d[j])
            assert E_d[j, a] - E_d[j, b] <= bound[j, a] + bound[j, b], (j, a, b)
            st["near_tie"] += 1
        assert c_o[j] == cand_o[j, best_o[j]]

    # ---- codes under the oracle's scales: clamp(rne(X/(rho c))) ----
    codes_d = D.codes_under(Xd, rho_o, act, rb, c_o)
    P = D.half_value(rho_o)[:, None] * D.half_value(c_o)[None, :]
    okp = act[:, None] & (P > 0)
    t = np.abs(np.where(okp, Xd / np.where(okp, P, 1.0), 0.0))
    tie = okp & (np.abs(t - np.floor(t) - 0.5) <= 2.0 ** -22 * (t + 1))
    st["code_tie"] += int(tie.sum())
    assert np.array_equal(codes_o[~tie & quant[:, None]], codes_d[~tie & quant[:, None]])

    # ---- end to end: the definition with its own scales ----
    ref = D.quantize_head(Xd, rb, w)
    assert np.array_equal(piv_o[~quant], ref["piv"][~quant])
    diff = quant[:, None] & (codes_o != ref["codes"])
    cdiff = c_o != ref["c"]
    rdiff = rho_o != ref["rho"]
    st["entries"] += int(quant.sum()) * dv
    st["codes_differ"] += int(diff.sum())
    st["c_differ"] += int(cdiff.sum())
    st["rho_differ"] += int(rdiff.sum())
    same_scales = ~rdiff[:, None] & ~cdiff[None, :]
    assert np.all(np.abs(codes_o[diff & same_scales].astype(np.int64)
                         - ref["codes"][diff & same_scales].astype(np.int64)) <= 1)


@pytest.mark.parametrize("name", ["gdn", "kda", "pool", "rollout"])
def test_stated_order_fit_matches_definition_fullsize(orc, name):
    st = dict(rows=0, rho_boundary=0, cands=0, cand_boundary=0, columns=0, close_pairs=0,
              near_tie=0, code_tie=0, entries=0, codes_differ=0, c_differ=0, rho_differ=0)
    for ora, h, X, rb, w in _cases(orc, name):
        _check(ora, h, X, rb, w, st)
    print(f"\n{name}: {st}")
    assert st["columns"] >= 2 * HEADS_PER_WORKLOAD * 128
    assert st["near_tie"] <= 1e-3 * st["columns"]
    assert st["codes_differ"] <= 1e-3 * st["entries"]
    assert st["c_differ"] <= 1e-3 * st["columns"]
    assert st["rho_differ"] <= 1e-3 * st["rows"]


def test_definition_half_rounding_is_exact():
    """numpy's float64 -> float16 conversion, which the definition reading
    uses for every scale, against exact rational rounding: random values and
    values one float64 ulp either side of binary16 midpoints."""
    from fractions import Fraction as Fr
    rng = np.random.default_rng(5)
    vals = list(np.exp(rng.uniform(np.log(2.0 ** -26), np.log(70000.0), 3000)))
    for k in range(1, 2047, 7):
        for e in (-24, -14, -3, 0, 5, 14):
            g = 2.0 ** (e - 10) if e >= -14 else 2.0 ** -24
            mid = (k + 0.5) * g if e >= -14 else (k % 1023 + 0.5) * g
            vals += [mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf)]
    for v in vals:
        if not (0 < v < 65520):
            continue
        x = Fr(float(v))
        if x < Fr(1, 2 ** 14):
            g = Fr(1, 2 ** 24)
        else:
            e = 0
            while Fr(2) ** (e + 1) <= x:
                e += 1
            while Fr(2) ** e > x:
                e -= 1
            g = Fr(2) ** (e - 10)
        q = x / g
        f = q.numerator // q.denominator
        rem = q - f
        n = f + 1 if rem > Fr(1, 2) or (rem == Fr(1, 2) and f % 2) else f
        want = min(n * g, Fr(65504))
        got = Fr(float(D.half_value(D.half_bits(v))))
        assert got == want, v


def test_definition_tie_rules():
    """The definition reading's discrete rules on hand-made values: equal
    objectives go to the larger alpha (the first candidate), codes round half
    to even and clamp at +-qmax, a positive scale never rounds to zero."""
    E = np.array([[3.0, 2.0, 2.0, 5.0, 2.0, 9.0, 9.0, 9.0],
                  [1.0, 1.0, 1.0, 1.0, 1.0, 1.0, 1.0, 1.0],
                  [4.0, 4.0, 4.0, 4.0, 4.0, 4.0, 4.0, 0.5]])
    assert list(D.argmin_first(E)) == [1, 0, 7]
    one = np.uint16(0x3C00)   # 1.0
    X = np.array([[2.5, -2.5, 3.5, 40.0, -0.5, 0.49]])
    codes = D.codes_under(X, np.array([one]), np.array([True]), np.array([6]),
                          np.full(6, one, np.uint16))
    assert list(codes[0]) == [2, -2, 4, 31, 0, 0]
    assert D.scale_bits(np.array([1e-12]))[0] == 1 and D.scale_bits(np.array([0.0]))[0] == 0
    assert np.all(D.candidates(np.array([0.0, 1.0]), 31.0)[0] == 0)
