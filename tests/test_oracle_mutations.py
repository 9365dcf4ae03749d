"""The oracle's pins catch plausible mistakes.

Each mutation below plants one mistake in a copy of oracle/stepq_oracle.c (a
flipped sign, a dropped term, a transposed index, a wrong rounding, a wrong
tie rule, a wrong bit order, ...).  The copy is built and the oracle's own pin
tests are run against it in a subprocess; every mutant must make at least one
of them fail.  A surviving mutant would mean a part of the oracle that nothing
other than itself checks.
"""

import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "stepq_oracle.c")
PINS = ["tests/test_oracle_half.py", "tests/test_oracle_pack.py", "tests/test_oracle_step.py",
        "tests/test_oracle_quant.py", "tests/test_oracle_alloc.py"]

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
