"""The oracle's pins catch plausible mistakes.

Each mutation below plants one mistake in a copy of oracle/stepq_oracle.c (a
flipped sign, a dropped term, a transposed index, a wrong rounding, a wrong
tie rule, a wrong bit order, ...) or of the Python parts of the oracle (the
bit allocation and the row-impact scores).  The copy is built and the
oracle's own pin tests are run against it in a subprocess; every mutant must
make at least one of them fail.  A surviving mutant would mean a part of the
oracle that nothing other than itself checks.
"""

import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "stepq_oracle.c")
PINS = ["tests/test_oracle_half.py", "tests/test_oracle_pack.py", "tests/test_oracle_step.py",
        "tests/test_oracle_quant.py", "tests/test_oracle_alloc.py", "tests/test_oracle_fullsize_fit.py"]

MUTATIONS = {
    "delta sign": ("delta = beta * (v[j] - u);", "delta = beta * (u - v[j]);"),
    "gate dropped from X": ("X[i * dv + j] = g * S[i * dv + j] + k[i] * delta;",
                            "X[i * dv + j] = S[i * dv + j] + k[i] * delta;"),
    "readout after requantisation": ("acc = acc + q[i] * X[i * dv + j];",
                                     "acc = acc + q[i] * S[i * dv + j];"),
    "row factor times sqrt(w)": ("float r = sqrtf(m) / sqrtf(pl->w[h * dk + i]);",
                                 "float r = sqrtf(m) * sqrtf(pl->w[h * dk + i]);"),
    "objective weight without rho": (
        "Aw[i] = (pl->w[h * dk + i] * orc_half_to_float(rho[i])) *\n"
        "                        (pl->w[h * dk + i] * orc_half_to_float(rho[i]));",
        "Aw[i] = pl->w[h * dk + i] * pl->w[h * dk + i];"),
    "ties to the smaller alpha": ("if (a == 0 || E < Ebest) {", "if (a == 0 || E <= Ebest) {"),
    "candidate grid": ("1.0f, 0.95f, 0.9f, 0.85f", "1.0f, 0.95f, 0.95f, 0.85f"),
    "codes truncated": ("float r = rintf(t);                           /* round half to even */",
                        "float r = truncf(t);"),
    "bits MSB-first": ("row[bit / 8] |= (uint8_t)(1u << (bit % 8));",
                       "row[bit / 8] |= (uint8_t)(0x80u >> (bit % 8));"),
    "scales transposed": ("(orc_half_to_float(rho[i]) * orc_half_to_float(c[j]));",
                          "(orc_half_to_float(rho[j]) * orc_half_to_float(c[i]));"),
    "half rounding truncates": ("r = rintf(a / step) * step;", "r = truncf(a / step) * step;"),
    "width factor inverted": ("kappa[i] = (float)qhi / (float)qmax[i];",
                              "kappa[i] = (float)qmax[i] / (float)qhi;"),
    "distortion sign": ("double e = (double)Xh[i * dv + j] - (double)S[i * dv + j];",
                        "double e = (double)Xh[i * dv + j] + (double)S[i * dv + j];"),
    "offset binary off by one": ("(uint32_t)(codes[i * dv + j] + (1 << (b - 1)))",
                                 "(uint32_t)(codes[i * dv + j] + (1 << (b - 1)) - 1)"),
    "qmax off by one": ("qmax[i] = (1 << (b - 1)) - 1;", "qmax[i] = (1 << (b - 1));"),
    "column max without the width factor": ("z = fabsf(X[i * dv + j]) * ikap[i];",
                                            "z = fabsf(X[i * dv + j]) * irho[i];"),
    "objective without the clamp": ("        if (q > two23 + (float)qmax[i])\n            q = two23 + (float)qmax[i];",
                                    "        if (0)\n            q = two23 + (float)qmax[i];"),
    "row factor over w, not sqrt(w)": ("float r = sqrtf(m) / sqrtf(pl->w[h * dk + i]);",
                                       "float r = sqrtf(m) / pl->w[h * dk + i];"),
    "objective weight not squared": (
        "Aw[i] = (pl->w[h * dk + i] * orc_half_to_float(rho[i])) *\n"
        "                        (pl->w[h * dk + i] * orc_half_to_float(rho[i]));",
        "Aw[i] = pl->w[h * dk + i] * orc_half_to_float(rho[i]);"),
    "objective scaled by c, not c^2": ("return (c * c) * ((P[0] + P[1]) + (P[2] + P[3]));",
                                       "return c * ((P[0] + P[1]) + (P[2] + P[3]));"),
    "uniform scale over qmax + 1": ("rho[i] = scale_half(m / (float)qmax[i]);",
                                    "rho[i] = scale_half(m / (float)(qmax[i] + 1));"),
    "codes clamped asymmetrically": ("if (r < -(float)qmax) r = -(float)qmax;",
                                     "if (r < -(float)qmax - 1.0f) r = -(float)qmax - 1.0f;"),
    "delta without beta": ("delta = beta * (v[j] - u);", "delta = (v[j] - u);"),
    "update without k": ("X[i * dv + j] = g * S[i * dv + j] + k[i] * delta;",
                         "X[i * dv + j] = g * S[i * dv + j] + delta;"),
    "projection without the gate": ("u = u + k[i] * (g * S[i * dv + j]);   /* (k^T D S)_j */",
                                    "u = u + k[i] * S[i * dv + j];   /* (k^T D S)_j */"),
    "half rounding ties away": ("r = rintf(a / step) * step;", "r = roundf(a / step) * step;"),
    "subnormal halves truncated": ("r = rintf(a * 0x1p24f) * 0x1p-24f;", "r = truncf(a * 0x1p24f) * 0x1p-24f;"),
    "reconstruction without the row scale": (
        "S[i * dv + j] = (float)codes[i * dv + j] *\n"
        "                                (orc_half_to_float(rho[i]) * orc_half_to_float(c[j]));",
        "S[i * dv + j] = (float)codes[i * dv + j] *\n"
        "                                (orc_half_to_float(c[j]));"),
    "row maximum of signed values": ("float ax = fabsf(X[i * dv + j]);", "float ax = X[i * dv + j];"),
    "non-finite rows not flagged": ("            if (bad) {\n                status |= ORC_STATUS_NONFINITE;",
                                    "            if (bad) {\n                status |= 0;"),
    "non-finite rows kept": ("            if (bad) {\n                status |= ORC_STATUS_NONFINITE;\n                m = 0.0f;",
                             "            if (bad) {\n                status |= ORC_STATUS_NONFINITE;\n                m = m;"),
    "pivot rows not flagged when non-finite": (
        "                if (!isfinite(x))\n                    status |= ORC_STATUS_NONFINITE;\n"
        "                piv[i * dv + j] = orc_float_to_half(x);",
        "                if (!isfinite(x))\n                    status |= 0;\n"
        "                piv[i * dv + j] = orc_float_to_half(x);"),
    "readout with k for q": ("acc = acc + q[i] * X[i * dv + j];", "acc = acc + k[i] * X[i * dv + j];"),
    "beta on the projection only": ("delta = beta * (v[j] - u);", "delta = v[j] - beta * u;"),
    "distortion not squared": ("row += e * e;", "row += fabs(e);"),
    "zero-column scale kept": ("                if (M == 0.0f) {\n                    c[j] = 0;",
                               "                if (M == 0.0f) {\n                    c[j] = 0x3c00;"),
    "halves big-endian": ("static void put_half(uint8_t *p, uint16_t h) { p[0] = (uint8_t)(h & 0xff); p[1] = (uint8_t)(h >> 8); }",
                          "static void put_half(uint8_t *p, uint16_t h) { p[1] = (uint8_t)(h & 0xff); p[0] = (uint8_t)(h >> 8); }"),
    "column scales before row scales": ("put_half(blob + pl->scale_off[h] + 2 * dk + 2 * j, c[j]);",
                                        "put_half(blob + pl->scale_off[h] + 2 * j, c[j]);"),
    "codes of a row packed from the wrong offset": ("put_bits(row, j * b, b, (uint32_t)(codes[i * dv + j] + (1 << (b - 1))));",
                                                    "put_bits(row, j * b + 1, b, (uint32_t)(codes[i * dv + j] + (1 << (b - 1))));"),
    "a positive scale may round to zero": ("    if (x > 0.0f && h == 0)\n        h = 1;",
                                           "    if (x > 0.0f && h == 0)\n        h = 0;"),
    "seven candidates": ("                for (a = 0; a < 8; a++) {\n                    uint16_t ca",
                         "                for (a = 0; a < 7; a++) {\n                    uint16_t ca"),
    "candidates over qmax of the row": ("uint16_t ca = scale_half((ALPHA[a] * M) / (float)qhi);",
                                        "uint16_t ca = scale_half((ALPHA[a] * M) / (float)qmax[0]);"),
}


def _run(name, old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation '{name}' does not apply"
    d = os.path.join(tmp, name.replace(" ", "_"))
    os.makedirs(d)
    msrc = os.path.join(d, "stepq_oracle.c")
    open(msrc, "w").write(src.replace(old, new))
    env = dict(os.environ, STEPQ_ORACLE_SRC=msrc, STEPQ_ORACLE_LIB=os.path.join(d, "lib.so"),
               PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode


# a harmless edit (a comment): the pins must pass on it, so that a caught
# mutant means a failed pin and not a harness that cannot pass
CONTROL = ("control", ("/* round half to even */", "/* nearest, ties to even */"))


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda kv: _run(kv[0], *kv[1], tmp), [CONTROL, *MUTATIONS.items()]))
    assert results[0] == ("control", 0), f"the unmutated copy fails its pins: {results[0]}"
    results = results[1:]
    survivors = [name for name, rc in results if rc == 0]
    errors = [(name, rc) for name, rc in results if rc not in (0, 1)]
    assert not errors, f"pin runs that did not complete: {errors}"
    assert not survivors, f"mutations no pin caught: {survivors}"


# mistakes in the Python parts of the oracle: (module, old, new)
PY_PINS = ["tests/test_oracle_alloc.py", "tests/test_oracle_impact.py", "tests/test_oracle_fullsize_fit.py"]
PY_MUTATIONS = {
    "lifetime weight without the geometric sum": (
        "allocation.py", "out[u] = 1.0 / (1.0 - np.exp(ell))", "out[u] = np.exp(ell)"),
    "log retention averaged over steps only": (
        "allocation.py", "ell = acc / (steps * rows)", "ell = acc / steps"),
    "pivots by lowest risk": (
        "allocation.py", "key=lambda u: (-risk[u], u)", "key=lambda u: (risk[u], u)"),
    "pivot risk at the widest width": ("allocation.py", "col = WIDTHS.index(budget)", "col = 2"),
    "bit budget off by one": ("allocation.py", "K = N * (budget - 4) // 2", "K = N * (budget - 4) // 2 + 1"),
    "ties to the wider width": ("allocation.py", "better = cand < best", "better = cand <= best"),
    "backtracking loses the budget": ("allocation.py", "        k -= o", "        k -= min(o, 1)"),
    "impact without the gate": ("impact.py", "om = g * (q[r, h, i] - beta[r, h] * k[r, h, i] * kq)",
                                "om = (q[r, h, i] - beta[r, h] * k[r, h, i] * kq)"),
    "impact with the wrong sign": ("impact.py", "om = g * (q[r, h, i] - beta[r, h] * k[r, h, i] * kq)",
                                   "om = g * (q[r, h, i] + beta[r, h] * k[r, h, i] * kq)"),
    "impact without beta": ("impact.py", "om = g * (q[r, h, i] - beta[r, h] * k[r, h, i] * kq)",
                            "om = g * (q[r, h, i] - k[r, h, i] * kq)"),
    "weights without the square root": ("impact.py", "np.sqrt(s / count).astype(np.float32)",
                                        "(s / count).astype(np.float32)"),
    "definition: objective weight not squared": (
        "definition.py", "w2 = np.asarray(w, np.float64) ** 2", "w2 = np.asarray(w, np.float64)"),
    "definition: ties to the smaller alpha": (
        "definition.py", "best = np.where(E[:, a] < E[np.arange(E.shape[0]), best], a, best)",
        "best = np.where(E[:, a] <= E[np.arange(E.shape[0]), best], a, best)"),
    "definition: candidate grid": ("definition.py", "(100 - 5 * a) / 100.0", "(100 - 4 * a) / 100.0"),
    "definition: row factor times sqrt(w)": (
        "definition.py", "r = np.sqrt(m) / np.sqrt(np.asarray(w, np.float64))",
        "r = np.sqrt(m) * np.sqrt(np.asarray(w, np.float64))"),
    "definition: codes truncated": ("definition.py", "q = np.clip(np.rint(t),", "q = np.clip(np.trunc(t),"),
    "definition: column max without the width factor": (
        "definition.py", "z = np.abs(X[active]) / rho[active, None] * (qhi / qmax[active])[:, None]",
        "z = np.abs(X[active]) / rho[active, None]"),
    "definition: half rounding through float32": (
        "definition.py", "return x.astype(np.float16).view(np.uint16)",
        "return x.astype(np.float32).astype(np.float16).view(np.uint16)"),
    "definition: reconstruction without the row scale": (
        "definition.py", "e = np.where(active[:, None], X - (rho[:, None] * ca[None, :]) * code, 0.0)",
        "e = np.where(active[:, None], X - ca[None, :] * code, 0.0)"),
}


def _run_py(name, module, old, new, tmp):
    """The pins run from a directory whose oracle package holds the mutated
    module; everything else is linked to the real files."""
    d = os.path.join(tmp, name.replace(" ", "_"))
    os.makedirs(os.path.join(d, "oracle"))
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f == "__pycache__":
            continue
        os.symlink(os.path.join(ROOT, "oracle", f), os.path.join(d, "oracle", f))
    src = open(os.path.join(ROOT, "oracle", module)).read()
    assert src.count(old) == 1, f"mutation '{name}' does not apply"
    os.remove(os.path.join(d, "oracle", module))
    open(os.path.join(d, "oracle", module), "w").write(src.replace(old, new))
    for f in ("tests", "workload.py", "quantized_delta_rule_decode_b200"):
        os.symlink(os.path.join(ROOT, f), os.path.join(d, f))
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", *PY_PINS, "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu"], cwd=d, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_planted_mistake_in_the_python_oracle_fails_a_pin():
    import oracle
    oracle.build()
    # control: an edit of a comment only
    control = ("control", ("allocation.py", "# backward recurrence over the remaining units",
                           "# the recurrence, from the last unit back"))
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda kv: _run_py(kv[0], *kv[1], tmp), [control, *PY_MUTATIONS.items()]))
    assert results[0] == ("control", 0), f"the unmutated copy fails its pins: {results[0]}"
    results = results[1:]
    survivors = [name for name, rc in results if rc == 0]
    errors = [(name, rc) for name, rc in results if rc not in (0, 1)]
    assert not errors, f"pin runs that did not complete: {errors}"
    assert not survivors, f"mutations no pin caught: {survivors}"
