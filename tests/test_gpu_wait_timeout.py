"""Every device wait of the library is bounded; this test makes one run out.

The readout and the fit + pack kernels wait on mbarriers for their
bulk-async staging copies.  A wait that exceeds its limit records
STEPQ_DEV_TIMEOUT in the pool's status word, gives copies in flight a second
bounded wait and skips the head, so the GPU stays usable.  The test hook
stepq_pool_set_test_faults makes both kernels issue no staging copy (nothing
is in flight, so no wait can be satisfied) with a 1 ms limit; the step must
then return with the status bit set, the pool, y and the workspace
untouched, and the next ordinary step on the same pool must be exact again.
No fault, trap or endless loop is involved: every wait ends at its limit.
"""

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, dev, lib, pool_to_host, rel_l2, step_tensors

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["gdn", "kda"])
def test_wait_runs_out_and_next_step_is_exact(name):
    import torch
    cfg = W.CONFIGS[name]
    pair = Pair(cfg)
    S = lib()
    R = 4
    slots_np = np.arange(R, dtype=np.int32)
    slots = dev(slots_np)
    X0 = W.initial_state(cfg, range(R))
    o = pair.ora.new_pool(R)
    assert pair.ora.pack(o, slots_np, X0) == 0
    pool = pair.gpu_pool(R)
    pool.buf.copy_(torch.from_numpy(o))
    ws = torch.full((S.stepq_workspace_bytes(pair.gpu, R) // 4,), 7.0, dtype=torch.float32, device="cuda")
    y = torch.full((R, cfg.heads, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    si = W.step_inputs(cfg, 0, pair.pin, range(R))
    t = step_tensors(cfg, si)
    side = torch.cuda.Stream()

    S.stepq_pool_set_test_faults(pool, S.TEST_NO_STAGING_COPY, 1000)
    S.stepq_decode_step(pair.gpu, pool, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws, None, side)
    torch.cuda.synchronize()
    assert S.stepq_get_status(pool) & S.DEV_TIMEOUT
    assert np.array_equal(pool_to_host(pool), o), "a timed-out step must leave the pool untouched"
    assert torch.isnan(y).all() and bool((ws == 7.0).all())

    # back to normal: the same pool steps exactly as the oracle does
    S.stepq_pool_set_test_faults(pool, 0, 0)
    S.stepq_clear_status(pool)
    S.stepq_decode_step(pair.gpu, pool, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws, None, side)
    torch.cuda.synchronize()
    assert S.stepq_get_status(pool) == 0
    yo = np.zeros((R, cfg.heads, cfg.d), np.float32)
    for r in range(R):
        for h in range(cfg.heads):
            off, nb = pair.ora.head_layout(h)
            b0 = r * pair.slot_bytes + off
            blob = o[b0:b0 + nb].copy()
            yo[r, h], _, st = pair.ora.step_head(h, blob, si.q[r, h], si.k[r, h], si.v[r, h],
                                                 si.beta[r, h], si.gate[r, h])
            assert st == 0
            o[b0:b0 + nb] = blob
    assert np.array_equal(pool_to_host(pool), o)
    assert rel_l2(y.cpu().numpy(), yo) <= 1e-5


def test_test_fault_arguments_are_checked():
    cfg = W.CONFIGS["tiny"]
    pair = Pair(cfg)
    S = lib()
    pool = pair.gpu_pool(1)
    for flags, us in ((2, 10), (1, 0), (1, 2_000_000)):
        with pytest.raises(S.StepqError) as e:
            S.stepq_pool_set_test_faults(pool, flags, us)
        assert e.value.code == S._ffi.ERR_INVALID
