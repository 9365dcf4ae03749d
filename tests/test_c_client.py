"""The header is plain C and the library links into a C program.

A C11 translation unit includes include/stepq.h (no C++), links
libstepq.so and calls the host-only entry points: the lifetime weight of a
constant gate g is the geometric series 1 / (1 - g) (hyper.ai summary,
"Method", lifetime-aware bit allocation), an allocation under a 4-bit
budget is all 4 bits, and a refused call sets a message for
stepq_last_error().  Needs gcc, no GPU."""

import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <math.h>
#include <stdio.h>
#include <string.h>
#include "stepq.h"

int main(void) {
    float gate[3 * 2 * 4];
    double weight[2], dist[2 * 3] = {4, 2, 1, 8, 4, 2};
    uint8_t bits[2];
    int i;
    for (i = 0; i < 3 * 2 * 4; ++i) gate[i] = i % 8 < 4 ? 0.5f : 0.75f;
    if (stepq_lifetime_weight(2, 3, 4, gate, weight) != STEPQ_OK) return 1;
    if (fabs(weight[0] - 2.0) > 1e-12 || fabs(weight[1] - 4.0) > 1e-12) return 2;
    if (stepq_allocate_bits(2, weight, dist, 4, 0, bits) != STEPQ_OK) return 3;
    if (bits[0] != 4 || bits[1] != 4) return 4;
    if (stepq_lifetime_weight(2, 3, 4, NULL, weight) != STEPQ_ERR_INVALID) return 5;
    if (strlen(stepq_last_error()) == 0) return 6;
    printf("ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_a_c_program_includes_the_header_and_links_the_library():
    from quantized_delta_rule_decode_b200 import build as B
    lib = B.build()
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "client.c")
        exe = os.path.join(tmp, "client")
        open(src, "w").write(PROGRAM)
        subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                               "-o", exe, lib, "-lm", f"-Wl,-rpath,{os.path.dirname(lib)}"])
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
        assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
