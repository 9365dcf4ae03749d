"""GPU fp32-state baseline step vs the oracle's (same update, unquantised).

The unquantised baseline is the FP32-state update the pages compare against
(rcap.io post, results paragraph: 2.91x faster state update than FP32).
"""

import numpy as np
import pytest

import oracle
import workload as W
from gpu_harness import dev, lib, rel_l2, step_tensors

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,R", [("tiny", 1), ("gdn", 4), ("kda", 3)])
def test_fp32_step_matches_oracle(name, R):
    import torch
    cfg = W.CONFIGS[name]
    p = W.make_plan(cfg)
    nslots = cfg.pool_slots if cfg.permute_slots else R
    slots = W.slot_indices(cfg)[:R] if cfg.permute_slots else np.arange(R, dtype=np.int32)
    S0 = np.zeros((nslots, cfg.heads, cfg.d, cfg.d), np.float32)
    S0[slots] = W.initial_state(cfg, range(R))
    Sg = dev(S0)
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    So = S0.copy()
    for step in range(3):
        si = W.step_inputs(cfg, step, p, range(R))
        t = step_tensors(cfg, si)
        y = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
        lib().stepq_fp32_step(Sg, dev(slots), t["q"], t["k"], t["v"], t["beta"], t["gate"], y,
                              cfg.gate_kind, dev_status=status)
        yo, st = oracle.fp32_step(So, slots, si.q, si.k, si.v, si.beta, si.gate, cfg.gate_kind)
        assert st == 0
        assert rel_l2(y.cpu().numpy(), yo) <= 1e-5
        assert rel_l2(Sg.cpu().numpy(), So) <= 1e-6
    assert int(status[0].item()) == 0


def test_fp32_bad_slot():
    import torch
    cfg = W.CONFIGS["tiny"]
    p = W.make_plan(cfg)
    Sg = dev(W.initial_state(cfg))
    before = Sg.clone()
    si = W.step_inputs(cfg, 0, p)
    t = step_tensors(cfg, si)
    y = torch.empty((1, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    lib().stepq_fp32_step(Sg, dev(np.array([3], np.int32)), t["q"], t["k"], t["v"], t["beta"], t["gate"],
                          y, cfg.gate_kind, dev_status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) & 1
    assert torch.equal(Sg, before)
