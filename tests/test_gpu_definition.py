"""The GPU's packed state against the quantiser's plain definition (float64).

The kernels take the same binary32 decisions as the oracle (other tests assert
identical bytes).  This test closes the chain to the definition itself
(``oracle/definition.py``: row factors, column maxima, the 8 candidates, the
impact-weighted objective and the codes in float64 with no evaluation order;
hyper.ai summary, Method, dual-axis fitting; rcap.io post, decode-step
pseudocode): on full-size heads of gdn and kda, packed from the seeded
initial state and after one decode step, at most 0.1% of the GPU's codes may
differ from the definition's, and outside rows or columns whose scale differs
only by one level -- the benchmark's tolerance for the state.
"""

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, dev, lib, pool_to_host, step_tensors
from oracle import definition as D

pytestmark = pytest.mark.gpu


def _compare(pair, h, blob, X, st):
    codes, piv, rho, c = pair.ora.unpack_codes(h, blob)
    rb = pair.row_bits[h]
    ref = D.quantize_head(X.astype(np.float64), rb, pair.pin.w[h],
                          head_pivot=bool(pair.cfg.unit_kind == W.UNIT_HEAD and rb[0] == 16))
    quant = rb != 16
    if not np.any(quant):
        assert np.array_equal(piv, ref["piv"])
        return
    assert np.array_equal(piv[~quant], ref["piv"][~quant])
    rdiff = rho != ref["rho"]
    cdiff = c != ref["c"]
    assert np.all(np.abs(rho.astype(np.int64) - ref["rho"].astype(np.int64)) <= 1)
    diff = quant[:, None] & (codes != ref["codes"])
    same = ~rdiff[:, None] & ~cdiff[None, :]
    assert np.all(np.abs(codes[diff & same].astype(np.int64) - ref["codes"][diff & same].astype(np.int64)) <= 1)
    st["entries"] += int(quant.sum()) * codes.shape[1]
    st["differ"] += int(diff.sum())
    st["cols"] += codes.shape[1]
    st["c_differ"] += int(cdiff.sum())


@pytest.mark.parametrize("name", ["gdn", "kda"])
def test_gpu_codes_match_the_definition(name):
    import torch
    cfg = W.CONFIGS[name]
    pair = Pair(cfg)
    S = lib()
    R = 6
    slots_np = np.arange(R, dtype=np.int32)
    slots = dev(slots_np)
    X0 = W.initial_state(cfg, range(R))
    pool = pair.gpu_pool(R)
    S.stepq_pack(pair.gpu, pool, slots, dev(X0))
    g0 = pool_to_host(pool)
    st = dict(entries=0, differ=0, cols=0, c_differ=0)
    for r in range(R):
        for h in range(cfg.heads):
            _compare(pair, h, pair.head_blob(g0, r, h), X0[r, h], st)
    # one step: the GPU requantises X = D S + k delta^T, which equals the
    # oracle's X bit for bit (delta is the plain definition's)
    si = W.step_inputs(cfg, 0, pair.pin, range(R))
    t = step_tensors(cfg, si)
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")
    y = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
    S.stepq_decode_step(pair.gpu, pool, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws)
    g1 = pool_to_host(pool)
    for r in range(R):
        for h in range(cfg.heads):
            blob = pair.head_blob(g0, r, h).copy()
            _, X1, status = pair.ora.step_head(h, blob, si.q[r, h], si.k[r, h], si.v[r, h], si.beta[r, h],
                                               si.gate[r, h])
            assert status == 0
            _compare(pair, h, pair.head_blob(g1, r, h), X1, st)
    assert S.stepq_get_status(pool) == 0
    print(f"\n{name}: {st}")
    assert st["differ"] <= 1e-3 * st["entries"]
    assert st["c_differ"] <= 1e-3 * st["cols"]
