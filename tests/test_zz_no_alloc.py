"""The allocation-free decode step (stepq_decode_step_static) against the
ordinary one (stepq_decode_step), through the C ABI.

Some callers cannot allocate device memory (a framework whose caching
allocator owns it all, a process that may not grow its device footprint, a
C caller with no allocator), so this entry point keeps its only scratch --
the delta vector passed from the readout kernel to the fit kernel -- in a
fixed device array inside the library.  Its results must equal those of the
ordinary entry point on the same inputs, call after call.  This file is
collected last so a stop-at-first-failure run has already run every other
test.
"""

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, dev, lib, pool_to_host, rel_l2, step_tensors

pytestmark = pytest.mark.gpu


def test_static_step_matches_decode_step_two_calls():
    import torch
    cfg = W.CONFIGS["gdn"]
    pair = Pair(cfg)
    S = lib()
    R = 8
    slots = dev(np.arange(R, dtype=np.int32))
    X0 = dev(W.initial_state(cfg, range(R)))
    pool_a, pool_b = pair.gpu_pool(R), pair.gpu_pool(R)
    S.stepq_pack(pair.gpu, pool_a, slots, X0)
    S.stepq_pack(pair.gpu, pool_b, slots, X0)
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    for call in range(2):
        si = W.step_inputs(cfg, call, pair.pin, range(R))
        t = step_tensors(cfg, si)
        ya = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
        yb = torch.empty_like(ya)
        S.stepq_decode_step(pair.gpu, pool_a, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"],
                            ya, ws, None, side)
        S.stepq_decode_step_static(pair.gpu, pool_b, slots, t["q"], t["k"], t["v"], t["beta"],
                                   t["gate"], yb, None, side)
        torch.cuda.synchronize()
        assert rel_l2(yb.cpu().numpy(), ya.cpu().numpy()) <= 1e-5
        assert np.array_equal(pool_to_host(pool_b), pool_to_host(pool_a))
    assert S.stepq_get_status(pool_a) == 0 and S.stepq_get_status(pool_b) == 0


def test_static_step_rejects_more_than_its_array():
    import torch
    cfg = W.CONFIGS["gdn"]
    pair = Pair(cfg)
    S = lib()
    R = S._ffi.STATIC_DELTA_FLOATS // (cfg.heads * cfg.d) + 1
    pool = pair.gpu_pool(R)
    slots = dev(np.arange(R, dtype=np.int32))
    z = torch.zeros((R, cfg.heads, cfg.d), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros((R, cfg.heads), dtype=torch.float32, device="cuda")
    y = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
    with pytest.raises(S.StepqError) as e:
        S.stepq_decode_step_static(pair.gpu, pool, slots, z, z, z, b, b, y)
    assert e.value.code == S._ffi.ERR_INVALID and "STEPQ_STATIC_DELTA_FLOATS" in str(e.value)
