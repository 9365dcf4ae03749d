"""Multi-step rollouts, GPU vs oracle, each side evolving its own state.

Both start from the same packed state (packed by the oracle) and take the
same seeded inputs every step (fresh q, k, v, beta per step).  The contract:
over a 256-step rollout the dequantised state's relative Frobenius drift
from the oracle's stays <= 1e-3.  The long rollout workload (128 requests x 16 heads, 4096 steps)
runs in full on the GPU, in the launch configuration bench.py times, and is
compared on a fixed subset of 2 requests x 16 heads.  Since the kernels
evaluate delta, X and the column objective in the oracle's order, the
rollouts stay identical, and the tests also check the packed bytes (every step for the
short rollouts) and the readout y of every step (relative L2 <= 1e-5, the
one-step bound).
"""

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, dev, lib, pool_to_host, rel_l2, rel_l2_worst_head, step_tensors

pytestmark = pytest.mark.gpu


def _rollout(name, steps, compare_reqs, gpu_reqs, mode=W.MODE_STEPQUANT, ub=None, every=32,
             bytes_every=None):
    import torch
    cfg = W.CONFIGS[name]
    pair = Pair(cfg, mode=mode, uniform_bits=ub)
    S = lib()
    R = gpu_reqs
    slots = np.arange(R, dtype=np.int32)
    o = pair.ora.new_pool(R)
    X0 = W.initial_state(cfg, range(R))
    pair.ora.pack(o, slots, X0)
    pool = pair.gpu_pool(R)
    pool.buf.copy_(torch.from_numpy(o))
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")
    y = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream()
    sl = dev(slots)
    Sg = torch.empty((R, cfg.heads, cfg.d, cfg.d), dtype=torch.float32, device="cuda")
    keys = [(r, h) for r in compare_reqs for h in range(cfg.heads)]
    ex = ThreadPoolExecutor(8)
    worst_drift, worst_y = 0.0, 0.0
    for step in range(steps):
        si = W.step_inputs(cfg, step, pair.pin, range(R))
        t = step_tensors(cfg, si)
        S.stepq_decode_step(pair.gpu, pool, sl, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws,
                            None, side)
        yo = {}

        def one(key):
            r, h = key
            off, nb = pair.ora.head_layout(h)
            b0 = r * pair.slot_bytes + off
            blob = o[b0:b0 + nb].copy()
            yy, _, _ = pair.ora.step_head(h, blob, si.q[r, h], si.k[r, h], si.v[r, h], si.beta[r, h],
                                          si.gate[r, h])
            o[b0:b0 + nb] = blob
            yo[key] = yy

        list(ex.map(one, keys))
        # the readout of every step, against the oracle's
        yg = y.cpu().numpy()
        worst_y = max(worst_y, rel_l2_worst_head(np.array([yg[r, h] for (r, h) in keys]),
                                                 np.array([yo[key] for key in keys])))
        if bytes_every and (step % bytes_every == bytes_every - 1 or step == steps - 1):
            # the packed slots, byte for byte: a transient divergence (one row
            # factor off by a half ulp for one step) cannot pass unseen
            gb = pool_to_host(pool)
            for r in compare_reqs:
                a, b = r * pair.slot_bytes, (r + 1) * pair.slot_bytes
                assert np.array_equal(gb[a:b], o[a:b]), f"step {step}: request {r} state differs"
        if step % every == every - 1 or step == steps - 1:
            S.stepq_unpack(pair.gpu, pool, sl, Sg)
            torch.cuda.synchronize()
            gS = Sg.cpu().numpy()
            oS, _ = pair.ora.unpack(o, slots)
            for r in compare_reqs:
                d = rel_l2(gS[r], oS[r])
                worst_drift = max(worst_drift, d)

    ex.shutdown()
    assert S.stepq_get_status(pool) == 0
    return worst_drift, worst_y


def test_rollout_tiny_256_steps():
    drift, ydiff = _rollout("tiny", 256, [0], 1, every=8, bytes_every=1)
    assert drift <= 1e-3, drift
    assert ydiff <= 1e-5, ydiff


def test_rollout_tiny_uniform8_256_steps():
    drift, ydiff = _rollout("tiny", 256, [0], 1, mode=W.MODE_UNIFORM, ub=8, every=16, bytes_every=1)
    assert drift <= 1e-3, drift
    assert ydiff <= 1e-5, ydiff


def test_rollout_kda_256_steps():
    """Per-key-row gates and widths (with FP16 pivot rows), 2 requests."""
    drift, ydiff = _rollout("kda", 256, [0, 1], 2, every=64, bytes_every=1)
    assert drift <= 1e-3, drift
    assert ydiff <= 1e-5, ydiff


@pytest.mark.slow
def test_rollout_long_4096_steps_subset():
    """128 requests x 16 heads on the GPU for 4096 steps; 2 x 16 compared."""
    drift, ydiff = _rollout("rollout", 4096, [0, 1], 128, every=256, bytes_every=256)
    assert drift <= 1e-3, drift
    assert ydiff <= 1e-5, ydiff
