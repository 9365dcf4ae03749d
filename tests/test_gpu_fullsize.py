"""Full-size workloads in the launch configuration bench.py times, checked on
sampled (request, head) pairs the oracle computes one by one.

The GPU packs and steps every request of the workload at once (readout on
the main stream, fit + pack on a side stream).  Requests are independent, so
the sampled requests get their exact seeded initial state while the others
get any synthetic state; the oracle packs and steps the sampled heads from
the seeded inputs alone, and both the packed initial state (bit-exact
contract) and one full step (readout rel-L2 <= 1e-5, <= 0.1% codes off by
one) are compared.
"""

import numpy as np
import pytest

import workload as W
from gpu_harness import (Pair, StepDiff, compare_pack, dev, lib, new_stats, pool_to_host, rel_l2,
                         rel_l2_worst_head)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,samples", [("gdn", 12), ("kda", 12), ("pool", 12)])
def test_fullsize_sampled(name, samples):
    import torch
    cfg = W.CONFIGS[name]
    pair = Pair(cfg)
    S = lib()
    R, H, d = cfg.requests, cfg.heads, cfg.d
    rng = np.random.default_rng(123)
    picks = sorted({(int(rng.integers(R)), int(rng.integers(H))) for _ in range(samples)})
    reqs = sorted({r for r, _ in picks})
    slots_np = W.slot_indices(cfg)
    slots = dev(slots_np)
    # initial state: seeded for the sampled requests, synthetic elsewhere
    X = torch.randn((R, H, d, d), dtype=torch.float32, device="cuda")
    X *= torch.exp(torch.randn((R, H, d, 1), device="cuda"))
    X0s = W.initial_state(cfg, reqs)
    for a, r in enumerate(reqs):
        X[r] = torch.from_numpy(X0s[a]).cuda()
    pool = pair.gpu_pool(cfg.pool_slots)
    S.stepq_pack(pair.gpu, pool, slots, X)
    del X
    g0 = pool_to_host(pool)
    # the oracle packs the sampled heads itself
    o = {}
    stats = new_stats()
    for r, h in picks:
        X0 = X0s[reqs.index(r), h]
        blob, st = pair.ora.quantize_head(h, X0)
        assert st == 0
        compare_pack(pair, h, pair.head_blob(g0, slots_np[r], h), blob, X0, stats)
        o[(r, h)] = blob                 # the oracle continues from its own packed state
    # one full-size step, two streams
    si = W.step_inputs(cfg, 0, pair.pin)
    dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
    q, k, v = (torch.from_numpy(a).to(dt).cuda() for a in (si.q, si.k, si.v))
    beta, gate = torch.from_numpy(si.beta).cuda(), torch.from_numpy(si.gate).cuda()
    y = torch.empty((R, H, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")
    S.stepq_decode_step(pair.gpu, pool, slots, q, k, v, beta, gate, y, ws, None, torch.cuda.Stream())
    torch.cuda.synchronize()
    g1 = pool_to_host(pool)
    yg = y.cpu().numpy()
    ys, yos = [], []
    diff = StepDiff()
    for r, h in picks:
        blob = o[(r, h)]
        yo, _, st = pair.ora.step_head(h, blob, si.q[r, h], si.k[r, h], si.v[r, h], si.beta[r, h],
                                       si.gate[r, h])
        assert st == 0
        ys.append(yg[r, h])
        yos.append(yo)
        diff.add(pair, h, pair.head_blob(g1, slots_np[r], h), blob, None)
    assert rel_l2(np.array(ys), np.array(yos)) <= 1e-5
    assert rel_l2_worst_head(np.array(ys), np.array(yos)) <= 1e-5
    diff.check(1e-3)
    assert S.stepq_get_status(pool) == 0
