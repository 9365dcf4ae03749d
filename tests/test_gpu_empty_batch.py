"""Empty batches: every entry point accepts n = 0, launches nothing and leaves
the pool as it was (status 0).  A serving loop calls the step with whatever
requests are active, which can be none."""

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, dev, lib, pool_to_host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "kda"])
def test_every_call_accepts_an_empty_batch(name):
    import torch
    cfg = W.CONFIGS[name]
    S = lib()
    pair = Pair(cfg)
    pool = pair.gpu_pool(2)
    S.stepq_pack(pair.gpu, pool, dev(np.arange(2, dtype=np.int32)), dev(W.initial_state(cfg, [0, 1])))
    before = pool_to_host(pool).copy()
    d, H = cfg.d, cfg.heads
    dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
    none = torch.empty(0, dtype=torch.int32, device="cuda")
    q = torch.empty((0, H, d), dtype=dt, device="cuda")
    beta = torch.empty((0, H), dtype=torch.float32, device="cuda")
    gate = torch.empty((0, H, d) if cfg.gate_kind == W.GATE_DIAG else (0, H), dtype=torch.float32,
                       device="cuda")
    y = torch.empty((0, H, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(1, S.stepq_workspace_bytes(pair.gpu, 0)), dtype=torch.uint8, device="cuda")
    X = torch.empty((0, H, d, d), dtype=torch.float32, device="cuda")
    S.stepq_pack(pair.gpu, pool, none, X)
    S.stepq_unpack(pair.gpu, pool, none, X)
    S.stepq_decode_readout(pair.gpu, pool, none, q, q, q, beta, gate, y, ws)
    S.stepq_decode_fitpack(pair.gpu, pool, none, q, gate, ws)
    S.stepq_decode_step(pair.gpu, pool, none, q, q, q, beta, gate, y, ws, None, torch.cuda.Stream())
    S.stepq_decode_step_static(pair.gpu, pool, none, q, q, q, beta, gate, y)
    hq = torch.empty((0, H, d), dtype=dt).pin_memory()
    S.stepq_decode_step_host(pair.gpu, pool, none, hq, hq, hq, beta.cpu(), gate.cpu(), y.cpu(), ws)
    torch.cuda.synchronize()
    assert np.array_equal(pool_to_host(pool), before)
    assert S.stepq_get_status(pool) == 0
