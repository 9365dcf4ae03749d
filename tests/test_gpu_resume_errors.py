"""Checkpoint / resume of the packed state, and faults injected on the host.

The state between tokens is the pool's bytes plus the plan (hyper.ai summary,
"Method", last paragraph: the state stays compressed between tokens).  Saving
the bytes and the plan's description, rebuilding both and continuing must give
exactly the bytes and readouts of an uninterrupted run.  Bad arguments are
refused on the host before any launch; a non-finite input is reported in the
pool's status word.  Nothing here faults, traps or hangs the GPU.
"""

import numpy as np
import pytest

import workload as W
from gpu_harness import Pair, dev, lib, pool_to_host, step_tensors

pytestmark = pytest.mark.gpu


def _steps(S, pair, pool, cfg, slots, ws, y, steps):
    out = []
    for step in steps:
        t = step_tensors(cfg, W.step_inputs(cfg, step, pair.pin, range(len(slots))))
        S.stepq_decode_step(pair.gpu, pool, dev(slots), t["q"], t["k"], t["v"], t["beta"], t["gate"],
                            y, ws)
        out.append(y.cpu().numpy().copy())
    return out


@pytest.mark.parametrize("name", ["tiny", "kda"])
def test_checkpoint_resume_is_bit_identical(name):
    import torch
    cfg = W.CONFIGS[name]
    S = lib()
    R = 2 if name == "kda" else 1
    slots = np.arange(R, dtype=np.int32)
    X0 = dev(W.initial_state(cfg, range(R)))
    y = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")

    pair = Pair(cfg)
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")
    pool = pair.gpu_pool(R)
    S.stepq_pack(pair.gpu, pool, dev(slots), X0)
    ys_full = _steps(S, pair, pool, cfg, slots, ws, y, range(6))
    full = pool_to_host(pool)

    a = Pair(cfg)
    pool_a = a.gpu_pool(R)
    S.stepq_pack(a.gpu, pool_a, dev(slots), X0)
    ys_a = _steps(S, a, pool_a, cfg, slots, ws, y, range(3))
    saved = pool_to_host(pool_a)              # checkpoint: the bytes + the plan description
    del pool_a, a
    b = Pair(cfg)                             # rebuilt from the same description
    pool_b = b.gpu_pool(R)
    pool_b.buf.copy_(torch.from_numpy(saved))
    ys_b = _steps(S, b, pool_b, cfg, slots, ws, y, range(3, 6))
    assert np.array_equal(pool_to_host(pool_b), full)
    for u, v in zip(ys_a + ys_b, ys_full):
        assert np.array_equal(u, v)
    assert S.stepq_get_status(pool_b) == 0


def test_host_checks_refuse_bad_arguments():
    import torch
    cfg = W.CONFIGS["gdn"]
    S = lib()
    R = 2
    pair, other = Pair(cfg), Pair(cfg)
    pool = pair.gpu_pool(R)
    slots = dev(np.arange(R, dtype=np.int32))
    t = step_tensors(cfg, W.step_inputs(cfg, 0, pair.pin, range(R)))
    y = torch.empty((R, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, R), dtype=torch.uint8, device="cuda")

    def refused(fn):
        with pytest.raises(S.StepqError) as e:
            fn()
        assert e.value.code == S._ffi.ERR_INVALID
        return str(e.value)

    # a q one element off 16-byte alignment
    qs = torch.empty(t["q"].numel() + 8, dtype=t["q"].dtype, device="cuda")
    q_off = qs[1:1 + t["q"].numel()].view(t["q"].shape)
    msg = refused(lambda: S.stepq_decode_step(pair.gpu, pool, slots, q_off, t["k"], t["v"], t["beta"],
                                              t["gate"], y, ws))
    assert "aligned" in msg
    # a pool created for another plan
    assert "another plan" in refused(lambda: S.stepq_decode_step(other.gpu, pool, slots, t["q"], t["k"],
                                                                 t["v"], t["beta"], t["gate"], y, ws))
    # a workspace one byte short
    assert "workspace" in refused(lambda: S.stepq_decode_step(pair.gpu, pool, slots, t["q"], t["k"], t["v"],
                                                              t["beta"], t["gate"], y, ws[:-1]))
    # pool buffers that are misaligned or too small
    buf = torch.zeros(2 * pair.slot_bytes + 256, dtype=torch.uint8, device="cuda")
    refused(lambda: S.stepq_pool_alloc(pair.gpu, 2, buf[16:]))
    refused(lambda: S.stepq_pool_alloc(pair.gpu, 3, buf))
    torch.cuda.synchronize()
    assert S.stepq_get_status(pool) == 0      # nothing was launched


def test_nonfinite_input_sets_status():
    import torch
    cfg = W.CONFIGS["tiny"]
    S = lib()
    pair = Pair(cfg)
    pool = pair.gpu_pool(1)
    slots = dev(np.zeros(1, np.int32))
    S.stepq_pack(pair.gpu, pool, slots, dev(W.initial_state(cfg, [0])))
    t = step_tensors(cfg, W.step_inputs(cfg, 0, pair.pin, [0]))
    t["v"][0, 1, 3] = float("nan")
    y = torch.empty((1, cfg.heads, cfg.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(S.stepq_workspace_bytes(pair.gpu, 1), dtype=torch.uint8, device="cuda")
    S.stepq_decode_step(pair.gpu, pool, slots, t["q"], t["k"], t["v"], t["beta"], t["gate"], y, ws)
    st = S.stepq_get_status(pool)
    assert st & S.DEV_NONFINITE
    S.stepq_clear_status(pool)
    assert S.stepq_get_status(pool) == 0
